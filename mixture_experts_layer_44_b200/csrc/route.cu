// Router on the CUDA cores (fp32 FMA), fused with softmax, warp-shuffle top-k
// and renormalisation: every fp32 batch, and bf16 batches of at most 64
// tokens and 64 experts (larger bf16 batches run on the tensor cores).
//
// DWDP-Triton-MoE-Inference-Engine README, "Router Module": router logits,
// routing probabilities, top-k expert indices, normalized routing weights.
// diffulex.moe API reference, "diffulex.moe.topk": NaiveTopKRouter.
//
// fp32 batches of more than 64 tokens (or more than 64 experts): a
// thread-block cluster of S CTAs (S <= 8) owns BT = 16*TT tokens and all E
// experts; CTA s of the cluster contracts its own slice of H.  Each CTA
// stages chunks of KC = 32 columns of x and W_gate (transposed, without bank
// conflicts) in double-buffered shared memory, prefetching the next chunk
// into registers while it computes the current one, and accumulates a
// TT-token x (EPAD/16)-expert register tile per thread (EPAD = 64, 128 or
// 256: E rounded up; TT = 8 for EPAD = 64, else 4).  Thread eg owns experts
// 64*(j/4) + 4*eg + (j%4): each of its float4 reads of W is part of 256
// contiguous bytes across the warp, free of bank conflicts.  The S partial
// logit tiles are then summed through distributed shared memory in a fixed
// rank order (deterministic, no global scratch): CTA s finalises tokens
// [s*BT/S, (s+1)*BT/S) of the tile, one warp per token, which adds the bias,
// writes the logits and selects the top k by k rounds of a warp arg-max on
// the key (logit descending, expert id ascending).
#include <cooperative_groups.h>
#include <float.h>

#include <algorithm>

#include "common.cuh"
#include "dispatch_cta.cuh"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace {

constexpr int KC = 32;    // H chunk
constexpr int NT = 256;   // threads per CTA
constexpr int MAX_S = 8;  // CTAs per cluster

// Eight elements at base + off (activations may come from the kernel before:
// read at L2, see moe::ld_prod).
template <bool BF16>
__device__ __forceinline__ void load8(const void* base, size_t off, bool ok, float* f) {
  if (!ok) {
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = 0.f;
    return;
  }
  if (BF16) {
    const uint4 q =
        moe::ld_prod(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + off));
    moe::unpack8(q, f);
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = moe::ld_prod(p), b = moe::ld_prod(p + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}


// Small batches (T <= 64 tokens, E <= 64 experts: decode): one CTA of 512
// threads (16 warps) per token.  The token's row of x is staged once in
// shared memory (fp32).  With EP = E rounded up to a power of two, each warp
// owns EPW = max(1, EP/16) experts and one of WPE = 16/min(EP,16) slices of
// H; lane l reads the 8-element vectors l, l+32, ... of the slice, so a
// warp's loads of a W_gate row are contiguous (512 bytes per instruction for
// bf16), with up to 16 loads in flight per lane.  Per (expert, slice) the
// lanes' partials are summed by a shuffle tree and warp 0 adds the slices in
// order, so the logits do not depend on timing.  Warp 0 then selects.
constexpr int NS = 512;   // threads per CTA of the small-batch router

// With FUSED, the router also dispatches: after its token is routed, each
// CTA makes its writes visible (__threadfence) and takes a ticket from a
// device counter; the CTA that takes the last ticket (no CTA ever waits for
// another) reads every token's selection at L2 and runs the single-CTA
// dispatch (per-warp counts, scan, stable scatter, and the gather of the rows
// when they total at most 128 KiB), then puts the counter back to zero for
// the next launch.
// With wsg (any launch of the small router), the shared expert's gate row is
// contracted with x as one more expert, E: its logit goes to sg[t] (no bias)
// and it takes no part in the top-k (diffulex.moe.layer, SharedExpertMLP).
struct SmallDispatch {
  int32_t* counter;            // zero before the launch; zero again after it
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  int32_t* packed_tok;
  float* packed_w;
  const uint4* x;              // null: no fused gather
  int row_vecs;
  uint4* x_packed;
  int32_t* status;
  const void* wsg;             // shared expert's gate row [H], or null
  float* sg;                   // its logit per token [T]
};

constexpr int kFusedRounds = 1;                       // N <= 16 warps x 32 = 512

template <int EP, bool BF16, bool FUSED>
__global__ void __launch_bounds__(NS) route_small_kernel(const void* xv,
                                                         const void* __restrict__ wv,
                                                         const float* __restrict__ bias, int H,
                                                         int E, int k, int renorm,
                                                         float* __restrict__ logits,
                                                         int32_t* ids, float* wout,
                                                         moe::GroupLimit gl, SmallDispatch dd) {
  constexpr int NWARP = NS / 32;
  constexpr int EPW = EP > NWARP ? EP / NWARP : 1;       // experts per warp
  constexpr int WPE = EP >= NWARP ? 1 : NWARP / EP;      // warps (H slices) per expert
  constexpr int GROUPS = NWARP / WPE;                     // expert e = group + GROUPS * i
  constexpr int Q = BF16 ? 1 : 2;                         // 16-byte words per 8 elements
  constexpr int BATCH = 16 / (EPW * Q);                   // vectors per expert in flight
  extern __shared__ __align__(16) float xs[];             // [H]
  __shared__ float part[EP][WPE];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = H / 8;
  const int slice = warp % WPE;
  const int group = warp / WPE;
  const int vs = slice * nvec / WPE, ve = (slice + 1) * nvec / WPE;
  const uint4* wb = reinterpret_cast<const uint4*>(wv);
  // One batch of W_gate vectors per lane; the loads are unconditional
  // (clamped to the slice's last vector) so that a whole batch is in flight
  // before the first FMA.
  uint4 wq[EPW][BATCH][Q];
  const int Etot = E + (dd.wsg != nullptr ? 1 : 0);       // rows: experts, then the gate
  auto load_w = [&](int vb) {
#pragma unroll
    for (int i = 0; i < EPW; ++i) {
      const int e = min(group + GROUPS * i, Etot - 1);
      const uint4* row = e < E ? wb + static_cast<size_t>(e) * nvec * Q
                               : static_cast<const uint4*>(dd.wsg);
#pragma unroll
      for (int j = 0; j < BATCH; ++j) {
        const int vc = min(vb + 32 * j, ve - 1);
#pragma unroll
        for (int q = 0; q < Q; ++q)
          wq[i][j][q] = moe::ld_nc_v4(row + static_cast<size_t>(vc) * Q + q);
      }
    }
  };
  // W_gate is a weight, never written by the kernel just before this one
  // (only this library's kernels let a successor start early, and none
  // writes it): the first batch is requested before waiting for that kernel.
  if (vs + lane < ve) load_w(vs + lane);
  moe::grid_dep_wait();
  for (int v = threadIdx.x; v < nvec; v += NS) {
    float f[8];
    load8<BF16>(xv, static_cast<size_t>(t) * H + v * 8, true, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) xs[v * 8 + j] = f[j];
  }
  __syncthreads();
  float acc[EPW];
#pragma unroll
  for (int i = 0; i < EPW; ++i) acc[i] = 0.f;
  for (int vb = vs + lane; vb < ve; vb += 32 * BATCH) {
    if (vb != vs + lane) load_w(vb);
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int v = vb + 32 * j;
      if (v >= ve) break;
      const float4 xa = *reinterpret_cast<const float4*>(&xs[v * 8]);
      const float4 xb = *reinterpret_cast<const float4*>(&xs[v * 8 + 4]);
#pragma unroll
      for (int i = 0; i < EPW; ++i) {
        float wf[8];
        if (BF16) {
          moe::unpack8(wq[i][j][0], wf);
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            wf[4 * q] = __uint_as_float(wq[i][j][q].x);
            wf[4 * q + 1] = __uint_as_float(wq[i][j][q].y);
            wf[4 * q + 2] = __uint_as_float(wq[i][j][q].z);
            wf[4 * q + 3] = __uint_as_float(wq[i][j][q].w);
          }
        }
        float a = acc[i];
        a = fmaf(xa.x, wf[0], a); a = fmaf(xa.y, wf[1], a);
        a = fmaf(xa.z, wf[2], a); a = fmaf(xa.w, wf[3], a);
        a = fmaf(xb.x, wf[4], a); a = fmaf(xb.y, wf[5], a);
        a = fmaf(xb.z, wf[6], a); a = fmaf(xb.w, wf[7], a);
        acc[i] = a;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < EPW; ++i) {
    float a = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    const int e = group + GROUPS * i;
    if (lane == 0 && e < EP) part[e][slice] = a;
  }
  __syncthreads();
  moe::grid_dep_launch();
  if (warp == 0) {
    constexpr int PER = 2;                     // experts lane, lane + 32
    float v[PER];
    bool live[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int ex = lane + 32 * j;
      live[j] = ex < E;
      float s = 0.f;
      if (live[j]) {
#pragma unroll
        for (int sl = 0; sl < WPE; ++sl) s += part[ex][sl];
        s += bias ? bias[ex] : 0.f;
        logits[static_cast<size_t>(t) * E + ex] = s;
      } else if (ex == E && dd.wsg != nullptr) {
#pragma unroll
        for (int sl = 0; sl < WPE; ++sl) s += part[ex][sl];
        dd.sg[t] = s;
      }
      v[j] = live[j] ? s : -FLT_MAX;
    }
    if (k > 0)
      moe::select_topk<PER>(v, live, k, renorm, ids + static_cast<size_t>(t) * k,
                            wout + static_cast<size_t>(t) * k, gl);
  }
  if constexpr (FUSED) {
    __shared__ int s_last;
    __shared__ int s_scan[moe::kMaxExperts];
    __syncthreads();                           // this token's ids and weights are written
    const bool one = gridDim.x == 1;           // a single token: no other CTA to wait for
    if (threadIdx.x == 0) {
      if (one) {
        s_last = 1;
      } else {
        __threadfence();
        s_last = atomicAdd(dd.counter, 1) == static_cast<int>(gridDim.x) - 1;
      }
    }
    __syncthreads();
    if (!s_last) return;
    if (!one) __threadfence();                 // every other token's writes are now visible
    // x is no longer needed: its shared memory holds the [NWARP][E] counts,
    // then the staged perm, packed_tok and packed_w
    int* wc = reinterpret_cast<int*>(xs);
    for (int i = threadIdx.x; i < NWARP * E; i += NS) wc[i] = 0;
    __syncthreads();
    moe::dispatch_cta<NWARP, kFusedRounds>(ids, wout, static_cast<int>(gridDim.x) * k, E, k,
                                           dd.counts, dd.offsets, dd.perm, dd.inv_perm,
                                           dd.packed_tok, dd.packed_w, dd.x, dd.row_vecs,
                                           dd.x_packed, dd.status, wc, s_scan, wc + NWARP * E);
    if (threadIdx.x == 0) *dd.counter = 0;
  }
}

// Token rows per thread: 8 when E <= 64 (more FMAs per shared-memory read),
// else 4.  A cluster then owns 16 * TT tokens.
template <int EPAD>
struct Tile {
  static constexpr int TT = EPAD == 64 ? 8 : 4;
  static constexpr int BT = 16 * TT;
  static constexpr int TE = EPAD / 16;
};

template <int EPAD, bool BF16>
__global__ void __launch_bounds__(NT) route_kernel(const void* xv,
                                                   const void* __restrict__ wv,
                                                   const float* __restrict__ bias, int T, int H,
                                                   int E, int k, int renorm, int kc_per_cta,
                                                   float* __restrict__ logits,
                                                   int32_t* __restrict__ ids,
                                                   float* __restrict__ wout,
                                                   moe::GroupLimit gl) {
  constexpr int TT = Tile<EPAD>::TT;
  constexpr int BTC = Tile<EPAD>::BT;        // tokens per cluster
  constexpr int TE = Tile<EPAD>::TE;         // experts per thread
  constexpr int LS = EPAD + 1;               // padded row of the logits tile
  constexpr int XV = BTC * (KC / 8) / NT;    // x vectors per thread per chunk (1 or 2)
  constexpr int WV = EPAD * (KC / 8) / NT;   // W_gate vectors per thread per chunk (1, 2 or 4)
  constexpr int XS = KC * BTC;               // one x buffer  [KC][BTC]
  constexpr int WS = KC * EPAD;              // one W buffer  [KC][EPAD]
  extern __shared__ __align__(16) float sm[];
  float* x_s = sm;                           // [2][KC][BTC]
  float* w_s = sm + 2 * XS;                  // [2][KC][EPAD]
  float* l_s = sm;                           // [BTC][LS] partial logits (after the loop)

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int eg = tid & 15;
  const int tg = tid >> 4;
  const int t0 = blockIdx.y * BTC;
  const int h_begin = rank * kc_per_cta * KC;
  const int h_end = min(H, h_begin + kc_per_cta * KC);

  float acc[TT][TE];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

  // Register staging of one chunk.  Vector i of the x chunk is token
  // (i % BTC), columns 8*(i / BTC) .. +8, so a warp stores 32 consecutive
  // tokens of one column group: no shared-memory bank conflicts.  W likewise.
  float xr[XV][8], wr[WV][8];
  auto fetch = [&](int h0) {
#pragma unroll
    for (int u = 0; u < XV; ++u) {
      const int i = tid + u * NT;
      const int t = i % BTC, hh = h0 + (i / BTC) * 8;
      load8<BF16>(xv, static_cast<size_t>(t0 + t) * H + hh, t0 + t < T && hh < h_end, xr[u]);
    }
#pragma unroll
    for (int u = 0; u < WV; ++u) {
      const int i = tid + u * NT;
      const int e = i % EPAD, hv = h0 + (i / EPAD) * 8;
      load8<BF16>(wv, static_cast<size_t>(e) * H + hv, e < E && hv < h_end, wr[u]);
    }
  };
  auto stash = [&](int b) {
    float* xs = x_s + b * XS;
    float* ws = w_s + b * WS;
#pragma unroll
    for (int u = 0; u < XV; ++u) {
      const int i = tid + u * NT;
      const int t = i % BTC, v = i / BTC;
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[(v * 8 + j) * BTC + t] = xr[u][j];
    }
#pragma unroll
    for (int u = 0; u < WV; ++u) {
      const int i = tid + u * NT;
      const int e = i % EPAD, v = i / EPAD;
#pragma unroll
      for (int j = 0; j < 8; ++j) ws[(v * 8 + j) * EPAD + e] = wr[u][j];
    }
  };

  moe::grid_dep_wait();
  if (h_begin < h_end) {
    fetch(h_begin);
    stash(0);
  }
  __syncthreads();
  int b = 0;
  for (int h0 = h_begin; h0 < h_end; h0 += KC, b ^= 1) {
    const bool more = h0 + KC < h_end;
    if (more) fetch(h0 + KC);                  // next chunk in flight during the FMAs
    const float* xs = x_s + b * XS;
    const float* ws = w_s + b * WS;
#pragma unroll 8
    for (int kk = 0; kk < KC; ++kk) {
      float xa[TT], wa[TE];
#pragma unroll
      for (int i = 0; i < TT; i += 4) {
        const float4 q = *reinterpret_cast<const float4*>(&xs[kk * BTC + tg * TT + i]);
        xa[i] = q.x; xa[i + 1] = q.y; xa[i + 2] = q.z; xa[i + 3] = q.w;
      }
#pragma unroll
      for (int j = 0; j < TE; j += 4) {             // experts 64*(j/4) + 4*eg + 0..3
        const float4 q = *reinterpret_cast<const float4*>(&ws[kk * EPAD + (j / 4) * 64 + eg * 4]);
        wa[j] = q.x; wa[j + 1] = q.y; wa[j + 2] = q.z; wa[j + 3] = q.w;
      }
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
    }
    if (more) stash(b ^ 1);                    // the other buffer was released by the last barrier
    __syncthreads();
  }

  moe::grid_dep_launch();
  // This CTA's partial logits tile (aliases the staging buffers, now idle).
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) l_s[(tg * TT + i) * LS + (j / 4) * 64 + eg * 4 + (j % 4)] = acc[i][j];
  cluster.sync();

  // Finalise tokens [rank*BTC/S, (rank+1)*BTC/S): one warp per token.
  constexpr int PER = EPAD / 32;
  const int warp = tid >> 5, lane = tid & 31;
  const int per_cta = (BTC + S - 1) / S;
  const int tl_end = min(BTC, (rank + 1) * per_cta);
  for (int tl = rank * per_cta + warp; tl < tl_end; tl += NT / 32) {
    const int t = t0 + tl;
    if (t >= T) break;
    float v[PER];
    bool live[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      live[j] = lane + 32 * j < E;
      v[j] = 0.f;
    }
    {
      // all ranks' partials in flight together, then summed in rank order
      float pv[MAX_S][PER];
#pragma unroll
      for (int r = 0; r < MAX_S; ++r) {
        if (r < S) {
          const float* rl = cluster.map_shared_rank(l_s, r);
#pragma unroll
          for (int j = 0; j < PER; ++j) pv[r][j] = live[j] ? rl[tl * LS + lane + 32 * j] : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < MAX_S; ++r)
        if (r < S)
#pragma unroll
          for (int j = 0; j < PER; ++j) v[j] += pv[r][j];
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
    moe::select_topk<PER>(v, live, k, renorm, ids + static_cast<size_t>(t) * k,
                          wout + static_cast<size_t>(t) * k, gl);
  }
  cluster.sync();   // no CTA leaves while another still reads its partial tile
}

template <int EPAD, bool BF16>
cudaError_t launch_t(const void* x, const void* W, const float* b, int T, int H, int E, int k,
                     int renorm, float* logits, int32_t* ids, float* w, moe::GroupLimit gl,
                     cudaStream_t s) {
  constexpr int BTC = Tile<EPAD>::BT;
  const size_t smem =
      sizeof(float) * std::max(2 * (KC * BTC + KC * EPAD), BTC * (EPAD + 1));
  auto fn = route_kernel<EPAD, BF16>;
  cudaError_t err = moe_host::ensure_smem(reinterpret_cast<const void*>(fn), (int)smem);
  if (err != cudaSuccess) return err;
  const int tiles = (T + BTC - 1) / BTC;
  const int chunks = (H + KC - 1) / KC;
  // Enough CTAs for ~4 per SM, never more than one chunk of H each.
  int S = (4 * moe_host::num_sms() + tiles - 1) / tiles;
  S = std::max(1, std::min({S, MAX_S, chunks}));
  const int kc_per_cta = (chunks + S - 1) / S;
  return moe_host::launch_pdl(fn, dim3(S, tiles, 1), dim3(NT, 1, 1), smem, s, S, x, W, b, T, H,
                              E, k, renorm, kc_per_cta, logits, ids, w, gl);
}

template <int EP, bool FUSED>
cudaError_t launch_small_ep(const void* x, const void* W, const float* b, int T, int H, int E,
                            int k, int renorm, bool bf, float* logits, int32_t* ids, float* w,
                            moe::GroupLimit gl, const SmallDispatch& dd, cudaStream_t s) {
  // The fused dispatch reuses the x row's shared memory for its [16][E]
  // counts and its three staged [512] arrays.
  const int smem = std::max(H, FUSED ? (NS / 32) * E + 3 * NS * kFusedRounds : 0) * 4;
  auto fn = bf ? route_small_kernel<EP, true, FUSED> : route_small_kernel<EP, false, FUSED>;
  cudaError_t e = moe_host::ensure_smem(reinterpret_cast<const void*>(fn), smem);
  if (e != cudaSuccess) return e;
  return moe_host::launch_pdl(fn, dim3(T), dim3(NS), smem, s, 0, x, W, b, H, E, k, renorm,
                              logits, ids, w, gl, dd);
}

template <bool FUSED>
cudaError_t launch_small(const void* x, const void* W, const float* b, int T, int H, int E, int k,
                         int renorm, bool bf, float* logits, int32_t* ids, float* w,
                         moe::GroupLimit gl, const SmallDispatch& dd, cudaStream_t s) {
  const int Er = E + (dd.wsg != nullptr ? 1 : 0);      // rows contracted (experts, gate)
  if (Er <= 1) return launch_small_ep<1, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  if (Er <= 2) return launch_small_ep<2, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  if (Er <= 4) return launch_small_ep<4, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  if (Er <= 8) return launch_small_ep<8, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  if (Er <= 16) return launch_small_ep<16, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  if (Er <= 32) return launch_small_ep<32, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
  return launch_small_ep<64, FUSED>(x, W, b, T, H, E, k, renorm, bf, logits, ids, w, gl, dd, s);
}

}  // namespace

namespace moe_host {

cudaError_t launch_route(const void* x, const void* W_gate, const float* bias, int T, int H,
                         int E, int k, int renormalize, int dtype, float* logits, int32_t* ids,
                         float* w, int32_t* status, cudaStream_t s, int n_groups,
                         int topk_groups) {
  const bool bf = dtype == MOE_BF16;
  const moe::GroupLimit gl{n_groups > 1 ? E / n_groups : E, n_groups > 1 ? n_groups : 1,
                           n_groups > 1 ? topk_groups : 1};
  if (T <= 64 && E <= 64 && H <= 32768)
    return launch_small<false>(x, W_gate, bias, T, H, E, k, renormalize, bf, logits, ids, w, gl,
                               SmallDispatch{}, s);
  if (bf)
    return launch_route_tc(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, status, s,
                           n_groups, topk_groups);
  if (E <= 64) return launch_t<64, false>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, gl, s);
  if (E <= 128) return launch_t<128, false>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, gl, s);
  if (E <= 256) return launch_t<256, false>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, gl, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_gated(const void* x, const void* W_gate, const float* bias,
                               const void* wsg, int T, int H, int E, int k, int renormalize,
                               int dtype, float* logits, int32_t* ids, float* w, float* sg,
                               int32_t* status, cudaStream_t s, int n_groups, int topk_groups) {
  const bool bf = dtype == MOE_BF16;
  const moe::GroupLimit gl{n_groups > 1 ? E / n_groups : E, n_groups > 1 ? n_groups : 1,
                           n_groups > 1 ? topk_groups : 1};
  const bool small = T <= 64 && E <= 64 && H <= 32768;   // launch_route's choice
  if (small && E + 1 <= 64) {
    SmallDispatch dd{};
    dd.wsg = wsg;
    dd.sg = sg;
    return launch_small<false>(x, W_gate, bias, T, H, E, k, renormalize, bf, logits, ids, w, gl,
                               dd, s);
  }
  if (bf && !small) {
    const cudaError_t e = launch_route_tc(x, W_gate, bias, T, H, E, k, renormalize, logits, ids,
                                          w, status, s, n_groups, topk_groups, wsg, sg);
    if (e != cudaErrorNotSupported) return e;
  }
  // two launches: the routed router, then the gate as one expert with no selection
  cudaError_t e = launch_route(x, W_gate, bias, T, H, E, k, renormalize, dtype, logits, ids, w,
                               status, s, n_groups, topk_groups);
  if (e != cudaSuccess) return e;
  return launch_route(x, wsg, nullptr, T, H, 1, 0, 0, dtype, sg, nullptr, nullptr, status, s);
}

bool route_dispatch_fits(int T, int H, int E, int k, bool gate) {
  return T >= 1 && T <= 64 && E >= 1 && E + (gate ? 1 : 0) <= 64 && H <= 32768 && k >= 1 &&
         k <= moe::kMaxTopK && T * k <= (NS / 32) * 32 * kFusedRounds;
}

cudaError_t launch_route_dispatch(const void* x, const void* W_gate, const float* bias, int T,
                                  int H, int E, int k, int renormalize, int dtype, float* logits,
                                  int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                                  int32_t* perm, int32_t* inv_perm, int32_t* packed_tok,
                                  float* packed_w, void* x_packed, int32_t* counter,
                                  int32_t* status, cudaStream_t s, int n_groups,
                                  int topk_groups, const void* wsg, float* sg) {
  const bool bf = dtype == MOE_BF16;
  const moe::GroupLimit gl{n_groups > 1 ? E / n_groups : E, n_groups > 1 ? n_groups : 1,
                           n_groups > 1 ? topk_groups : 1};
  const int row_bytes = H * (bf ? 2 : 4);
  const bool fuse_gather = x_packed != nullptr &&
                           static_cast<size_t>(T) * k * row_bytes <= (static_cast<size_t>(128) << 10);
  const SmallDispatch dd{counter, counts, offsets, perm, inv_perm, packed_tok, packed_w,
                         fuse_gather ? static_cast<const uint4*>(x) : nullptr, row_bytes / 16,
                         static_cast<uint4*>(x_packed), status, wsg, sg};
  cudaError_t e = launch_small<true>(x, W_gate, bias, T, H, E, k, renormalize, bf, logits, ids, w,
                                     gl, dd, s);
  if (e != cudaSuccess || x_packed == nullptr || fuse_gather) return e;
  return launch_gather(x, packed_tok, offsets, 0, E, T * k, H, dtype, x_packed, status, s);
}

}  // namespace moe_host
