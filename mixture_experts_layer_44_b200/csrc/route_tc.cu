// Router, bf16 batches: the gating GEMM on the 5th-generation tensor cores,
// fused with softmax, top-k and renormalisation.
//
// DWDP-Triton-MoE-Inference-Engine README, "Router Module": router logits,
// routing probabilities, top-k expert indices, normalized routing weights.
// diffulex.moe API reference, "diffulex.moe.topk": NaiveTopKRouter.
//
// logits = x W_gate^T is a dense [T,H] x [H,E] contraction with E <= 256, so
// it runs as tcgen05 MMAs of M = 128 tokens x N = EPAD experts (E rounded up
// to 32, 64, 128 or 256) per 16-wide step of H.  A bf16 x bf16 product is
// exact in fp32; the products are summed in fp32 in TMEM.
//
// A thread-block cluster of S CTAs (S <= 8) owns one tile of 128 tokens and
// CTA s contracts its own slice of H, in blocks of 64 columns that TMA brings
// into shared memory (128-byte swizzle; rows past T and experts past E read
// as zeros).  Successive blocks of the slice go round-robin to NCH separate
// accumulators in TMEM, so no fp32 chain adds more than 1/NCH of the slice;
// the epilogue adds the NCH chains in a fixed order into the CTA's partial
// logit tile in shared memory.  The S partial tiles are then summed through
// distributed shared memory in rank order (deterministic, no global scratch)
// and CTA s finalises its share of the tile's tokens, one warp per token (two
// tokens per pass): bias, logits, top-k on (logit descending, expert id
// ascending), softmax weights (renormalised or not).
//
// CTA = 8 warps: one lane of warp 0 issues the TMA loads, one lane of warp 1
// owns TMEM and issues the MMAs; then all 8 warps read the accumulators
// (warp w: TMEM lanes 32*(w%4) .. +31, column half w/4) and finalise tokens.
// With a shared expert's gate row (wsg, bf16 [H]; diffulex.moe.layer,
// SharedExpertMLP) its logit x . wsg is contracted in the same launch: the
// CTA's slice of wsg is staged in shared memory, warps 2-5 (one thread per
// token row, idle otherwise until the epilogue) read each stage's x tile
// after the TMA lands it and add 64 products per row in fp32, and the stage
// is released only once they and the MMAs are done with it.  Each CTA's
// partial goes into column E of its partial tile (a padding column: E <
// EPAD), so the cluster sums it with the logits; it takes no part in the
// selection and goes to sg[t] without bias.
//
// Every wait is bounded; one that runs out reports MOE_ERR_TIMEOUT in the
// status word and the CTA still takes part in both cluster barriers, so its
// peers finish too.  The stage-ring waits are bounded by `wait_ns` (a test
// hook can shorten it); the drain of issued copies and the wait for the
// issued MMAs (accf) always keep the full budget.
#include <cooperative_groups.h>
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "select.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

namespace cg = cooperative_groups;

namespace {

constexpr int RBM = 128;                  // tokens per tile (MMA M)
constexpr int RBK = 64;                   // H per pipeline stage: one 128-byte swizzle row
constexpr int RNT = 256;                  // threads per CTA
constexpr int RMAX_S = 8;                 // CTAs per cluster (portable limit)
constexpr int RMAX_STAGES = 8;
constexpr size_t RSTAGE_BUDGET = 144 * 1024;   // pipeline bytes: one CTA per SM
constexpr int RGATE_KB = 256;             // k-blocks of wsg a CTA can stage (32 KB)

template <int EPAD>
struct RCfg {
  static constexpr int A_BYTES = RBM * RBK * 2;
  static constexpr int B_BYTES = EPAD * RBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int LS = EPAD + 1;                        // padded row of the partial tile
  static constexpr size_t TILE_BYTES = sizeof(float) * RBM * LS;
  static constexpr size_t BUF_BYTES = TILE_BYTES > RSTAGE_BUDGET ? TILE_BYTES : RSTAGE_BUDGET;
  static constexpr int STAGES_FIT = static_cast<int>(BUF_BYTES / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT < RMAX_STAGES ? STAGES_FIT : RMAX_STAGES;
  static constexpr int NCH = EPAD >= 256 ? 1 : (EPAD == 128 ? 2 : 4);   // accumulator chains
  static constexpr uint32_t TMEM_COLS = NCH * EPAD;          // 128, 256, 256, 256
  static constexpr uint32_t IDESC = moe::idesc_bf16_f32(RBM, EPAD);
};

struct RCtl {
  uint64_t full[RMAX_STAGES];
  uint64_t empty[RMAX_STAGES];
  uint64_t accf;          // all MMAs of this CTA have completed
  uint32_t tmem_base;
  int abort;
  int gstop;              // the gate warps stop (their waiting thread timed out)
};

template <int EPAD>
constexpr size_t smem_bytes(bool gate) {
  return 1024 + RCfg<EPAD>::BUF_BYTES + (sizeof(RCtl) + 127) / 128 * 128 +
         (gate ? static_cast<size_t>(RGATE_KB) * RBK * 2 : 0);
}

__device__ __forceinline__ void set_abort(RCtl& c, int32_t* status) {
  moe::report(status, MOE_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c.abort) = 1;
}

template <int EPAD>
__global__ void __launch_bounds__(RNT, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmW, const float* __restrict__ bias,
                    int T, int E, int k, int renorm, int kblocks, float* __restrict__ logits,
                    int32_t* __restrict__ ids, float* __restrict__ wout, int32_t* status,
                    moe::GroupLimit gl, uint64_t wait_ns, const __nv_bfloat16* wsg,
                    float* __restrict__ sg, int H) {
  using C = RCfg<EPAD>;
  constexpr int LS = C::LS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  RCtl& c = *reinterpret_cast<RCtl*>(smem + C::BUF_BYTES);
  // the staged slice of the gate row (gate only)
  __nv_bfloat16* g_s = reinterpret_cast<__nv_bfloat16*>(
      smem + C::BUF_BYTES + (sizeof(RCtl) + 127) / 128 * 128);
  const bool gate = wsg != nullptr;
  float* l_s = reinterpret_cast<float*>(smem);   // after the main loop: [RBM][LS] partial logits

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int t0 = static_cast<int>(blockIdx.x / S) * RBM;
  const int kb0 = rank * kblocks / S;
  const int kb1 = (rank + 1) * kblocks / S;
  const int nkb = kb1 - kb0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      moe::mbar_init(moe::smem_addr(&c.full[s]), 1);
      moe::mbar_init(moe::smem_addr(&c.empty[s]), gate ? 2 : 1);   // MMAs (+ gate warps)
    }
    moe::mbar_init(moe::smem_addr(&c.accf), 1);
    c.abort = 0;
    moe::fence_barrier_init();
    moe::prefetch_tmap(&tmX);
    moe::prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    moe::tmem_alloc(moe::smem_addr(&c.tmem_base), C::TMEM_COLS);
    moe::tmem_relinquish();
  }
  if (gate && warp >= 2 && warp < 6) {
    // wsg is a weight (never the previous kernel's output): staged before the wait
    // (columns past H, in a last partial k-block, stay zero like the x tile's)
    const uint4* src = reinterpret_cast<const uint4*>(wsg + static_cast<size_t>(kb0) * RBK);
    uint4* dst = reinterpret_cast<uint4*>(g_s);
    for (int i = threadIdx.x - 64; i < nkb * RBK / 8; i += 128)
      dst[i] = kb0 * RBK + i * 8 < H ? moe::ld_nc_v4(src + i) : make_uint4(0, 0, 0, 0);
  }
  moe::grid_dep_wait();        // x may be the previous kernel's output
  moe::tc_fence_before();
  __syncthreads();
  moe::tc_fence_after();
  const uint32_t tmem = c.tmem_base;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer ---
    int stage = 0;
    uint32_t phase = 0;
    int issued[C::STAGES] = {};
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!moe::mbar_wait(moe::smem_addr(&c.empty[stage]), phase ^ 1, wait_ns)) {
        set_abort(c, status);
        break;
      }
      const uint32_t fb = moe::smem_addr(&c.full[stage]);
      const uint32_t sa = moe::smem_addr(smem + stage * C::STAGE_BYTES);
      moe::mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
      moe::tma_load_2d(sa, &tmX, fb, kb * RBK, t0);
      moe::tma_load_2d(sa + C::A_BYTES, &tmW, fb, kb * RBK, 0);
      ++issued[stage];
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
    // Drain: every load issued has landed before the buffers are reused.
    for (int s = 0; s < C::STAGES; ++s)
      if (issued[s] > 0) moe::mbar_wait(moe::smem_addr(&c.full[s]), (issued[s] - 1) & 1);
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA ---
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      if (!moe::mbar_wait(moe::smem_addr(&c.full[stage]), phase, wait_ns)) {
        set_abort(c, status);
        break;
      }
      moe::tc_fence_after();
      const uint32_t d = tmem + static_cast<uint32_t>((i % C::NCH) * EPAD);
      const uint32_t sa = moe::smem_addr(smem + stage * C::STAGE_BYTES);
#pragma unroll
      for (int kk = 0; kk < RBK / 16; ++kk) {
        const uint64_t ad = moe::sw128_kmajor_desc(sa + kk * 32);
        const uint64_t bd = moe::sw128_kmajor_desc(sa + C::A_BYTES + kk * 32);
        moe::tc_mma_f16(d, ad, bd, C::IDESC, (i >= C::NCH || kk > 0) ? 1u : 0u);
      }
      moe::tc_commit(moe::smem_addr(&c.empty[stage]));
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
    moe::tc_commit(moe::smem_addr(&c.accf));   // arrives once every MMA above has completed
  }
  // Gate: thread r of warps 2-5 adds row r of every landed x tile times the
  // staged wsg block (chunk j of row r sits at j ^ (r & 7): the 128-byte swizzle).
  float gacc = 0.f;
  if (gate && warp >= 2 && warp < 6) {
    const int r = threadIdx.x - 64;
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      // one thread waits (bounded) and tells the others through the named
      // barrier, so that all 128 leave the loop together
      if (r == 0) {
        const bool landed = moe::mbar_wait(moe::smem_addr(&c.full[stage]), phase, wait_ns);
        if (!landed) set_abort(c, status);
        *reinterpret_cast<volatile int*>(&c.gstop) = landed ? 0 : 1;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (*reinterpret_cast<volatile int*>(&c.gstop) != 0) break;
      moe::mbar_wait(moe::smem_addr(&c.full[stage]), phase, wait_ns);   // completed: returns
      const uint4* xr = reinterpret_cast<const uint4*>(smem + stage * C::STAGE_BYTES + r * 128);
      const uint4* wr = reinterpret_cast<const uint4*>(g_s + i * RBK);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float xf[8], wf[8];
        moe::unpack8(xr[j ^ (r & 7)], xf);
        moe::unpack8(wr[j], wf);
#pragma unroll
        for (int e = 0; e < 8; ++e) gacc = fmaf(xf[e], wf[e], gacc);
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");   // the four gate warps have read it
      if (r == 0) moe::mbar_arrive(moe::smem_addr(&c.empty[stage]));
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  __syncwarp();

  // ------------------------------------------- partial logits of this slice ---
  bool ok = moe::mbar_wait(moe::smem_addr(&c.accf), 0);
  if (!ok) set_abort(c, status);
  moe::tc_fence_after();
  __syncthreads();   // the producer has drained: no copy still writes the stage buffers
  ok = __all_sync(0xffffffffu, ok && *reinterpret_cast<volatile int*>(&c.abort) == 0);
  {
    constexpr int HALF = EPAD / 2;                 // accumulator columns per warp
    const int q = warp & 3;                        // TMEM lane quarter of this warp
    const int row = q * 32 + lane;
    const int nch = nkb < C::NCH ? nkb : C::NCH;   // chains that received a block
    const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16);
    if (ok) {
#pragma unroll 1
      for (int c0 = (warp >> 2) * HALF; c0 < (warp >> 2) * HALF + HALF; c0 += 16) {
        uint32_t a[16];
        float v[16];
        moe::tmem_ld16(tl + c0, a);
        moe::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(a[j]);
#pragma unroll
        for (int ch = 1; ch < C::NCH; ++ch) {     // fixed order
          if (ch < nch) {
            moe::tmem_ld16(tl + static_cast<uint32_t>(ch * EPAD + c0), a);
            moe::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(a[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) l_s[row * LS + c0 + j] = v[j];
      }
    } else {
      for (int c0 = (warp >> 2) * HALF; c0 < (warp >> 2) * HALF + HALF; ++c0)
        l_s[row * LS + c0] = 0.f;
    }
  }
  if (gate) {
    __syncthreads();                               // the tile's column E is written
    if (warp >= 2 && warp < 6) l_s[(threadIdx.x - 64) * LS + E] = ok ? gacc : 0.f;
  }
  moe::grid_dep_launch();
  moe::tc_fence_before();
  cluster.sync();
  moe::tc_fence_after();
  if (warp == 1) moe::tmem_dealloc(tmem, C::TMEM_COLS);

  // ---------------- finalise tokens [rank*RBM/S, (rank+1)*RBM/S) of the tile ---
  // One warp per token, lanes over experts, two tokens per pass (independent
  // reduction chains): add the S partials in rank order and the bias, write
  // the logits, select the top k and compute the weights.
  constexpr int PER = EPAD / 32;
  constexpr int NW = RNT / 32;
  const int per_cta = (RBM + S - 1) / S;
  const int tl_begin = rank * per_cta;
  const int tl_end = min(min(RBM, tl_begin + per_cta), T - t0);
  float bl[PER];
  bool live[PER], gcol[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    live[j] = e < E;
    gcol[j] = gate && e == E;                      // the shared gate's column
    bl[j] = (bias != nullptr && live[j]) ? bias[e] : 0.f;
  }
  for (int tl = tl_begin + warp; tl < tl_end; tl += 2 * NW) {
    const bool has_b = tl + NW < tl_end;
    const int rows[2] = {tl, has_b ? tl + NW : tl};
    float v[2][PER];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int j = 0; j < PER; ++j) v[n][j] = 0.f;
#pragma unroll
    for (int r = 0; r < RMAX_S; ++r) {
      if (r < S) {
        const float* rl = cluster.map_shared_rank(l_s, r);
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int j = 0; j < PER; ++j)
            v[n][j] += (live[j] || gcol[j]) ? rl[rows[n] * LS + lane + 32 * j] : 0.f;
      }
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const size_t t = static_cast<size_t>(t0 + rows[n]);
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        if (gcol[j] && (n == 0 || has_b)) sg[t] = v[n][j];
        v[n][j] += bl[j];
        if (live[j] && (n == 0 || has_b)) logits[t * E + lane + 32 * j] = v[n][j];
      }
    }
    if (k > 0) {
      const size_t ta = static_cast<size_t>(t0 + rows[0]) * k;
      const size_t tb = static_cast<size_t>(t0 + rows[1]) * k;
      int32_t* const it[2] = {ids + ta, has_b ? ids + tb : nullptr};
      float* const wt[2] = {wout + ta, has_b ? wout + tb : nullptr};
      moe::select_topk_n<PER, 2>(v, live, k, renorm, it, wt, gl);
    }
  }
  cluster.sync();   // no CTA leaves while another still reads its partial tile
}

template <int EPAD>
cudaError_t launch_t(const void* x, const void* W, const float* b, int T, int H, int E, int k,
                     int renorm, float* logits, int32_t* ids, float* w, int32_t* status,
                     moe::GroupLimit gl, cudaStream_t s, const void* wsg, float* sg) {
  auto fn = route_tc_kernel<EPAD>;
  const size_t smem = smem_bytes<EPAD>(wsg != nullptr);
  cudaError_t err = moe_host::ensure_smem(reinterpret_cast<const void*>(fn), (int)smem);
  if (err != cudaSuccess) return err;
  CUtensorMap mx, mw;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(H) * 2};
    const cuuint32_t box[2] = {RBK, RBM};
    if (!moe_host::encode_bf16_sw128(&mx, x, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(E)};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(H) * 2};
    const cuuint32_t box[2] = {RBK, EPAD};
    if (!moe_host::encode_bf16_sw128(&mw, W, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  const int tiles = (T + RBM - 1) / RBM;
  const int kblocks = (H + RBK - 1) / RBK;
  // One wave: as many H-slices per tile as the SMs allow, at least one block each.
  int S = moe_host::num_sms() / tiles;
  S = std::max(1, std::min({S, RMAX_S, kblocks}));
  if (wsg != nullptr && (kblocks + S - 1) / S > RGATE_KB) return cudaErrorNotSupported;
  return moe_host::launch_pdl(fn, dim3(S * tiles, 1, 1), dim3(RNT, 1, 1), smem, s, S, mx, mw, b,
                              T, E, k, renorm, kblocks, logits, ids, w, status, gl,
                              moe_host::main_wait_budget_ns(),
                              static_cast<const __nv_bfloat16*>(wsg), sg, H);
}

}  // namespace

namespace moe_host {

cudaError_t launch_route_tc(const void* x, const void* W_gate, const float* bias, int T, int H,
                            int E, int k, int renormalize, float* logits, int32_t* ids, float* w,
                            int32_t* status, cudaStream_t s, int n_groups, int topk_groups,
                            const void* wsg, float* sg) {
  const moe::GroupLimit gl{n_groups > 1 ? E / n_groups : E, n_groups > 1 ? n_groups : 1,
                           n_groups > 1 ? topk_groups : 1};
  const int Er = E + (wsg != nullptr ? 1 : 0);   // the gate takes column E (a padding column)
  if (Er <= 32) return launch_t<32>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, status, gl, s, wsg, sg);
  if (Er <= 64) return launch_t<64>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, status, gl, s, wsg, sg);
  if (Er <= 128) return launch_t<128>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, status, gl, s, wsg, sg);
  if (Er <= 256) return launch_t<256>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, status, gl, s, wsg, sg);
  return cudaErrorNotSupported;
}

}  // namespace moe_host
