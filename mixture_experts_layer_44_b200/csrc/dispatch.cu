// Dispatcher: token-major routing assignments -> expert-major layout.
//
// DWDP-Triton-MoE-Inference-Engine README, "Dispatcher Module": per-expert
// counts, expert offsets, token permutation, inverse permutation, packed
// token indices, packed routing weights; "Executor Module": gather token
// activations for the expert ranges.  Assignment f = t*k + j (row-major
// [T, k], the flat order of metrale's ep_dispatch.rs).
//
// Small batches (N <= 2048 assignments) take one CTA of 32 warps through
// count, scan and scatter in a single launch (the same warp-slice algorithm
// as below), and also gather the rows when they total at most 128 KiB
// (decode); larger gathers use the bulk-copy kernel.  Larger N takes three launches:
//   count   -- each CTA owns 1024 (N <= 65536) or 2048 consecutive
//              assignments; each warp owns a contiguous eighth of them and
//              counts it per expert with
//              __match_any_sync (one shared-memory add per distinct expert
//              in a 32-lane round, no atomics); CTA totals go to ws[b][e].
//   scatter -- each CTA reads the whole table: counts[e] = sum_b ws[b][e],
//              offsets = their exclusive scan over e (written by CTA 0), and
//              its own first position for expert e, offsets[e] +
//              sum_{b' < b} ws[b'][e]; it recounts its slice per warp, turns
//              the counts into per-warp bases, and walks its assignments in
//              order; inside a
//              round a lane's rank among equal experts is the popcount of
//              the lower lanes in its match mask.  Positions therefore grow
//              with f inside an expert: the order is stable (bit-exact).
//              The CTA's entries are staged in shared memory in expert
//              order and stored in runs of consecutive positions.
//   gather  -- x_packed[p] = x[packed_tok[p]] with bulk asynchronous copies
//              (global -> shared -> global on the TMA engine), one issuing
//              lane per warp, a 4-row ring per warp.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "common.cuh"
#include "dispatch_cta.cuh"
#include "sm100_ptx.cuh"

namespace {

// Assignments per CTA of the count and scatter kernels: 1024 up to
// CHUNK_SMALL_MAX assignments (the builder's 8192 on eight CTAs instead of
// four: dispatch 31.6 -> 28.5 us in the layer step), 2048 above (a longer
// per-expert scan over twice the CTAs cost Qwen3 ~2 us).
constexpr int CHUNK = 2048;
constexpr int CHUNK_SMALL = 1024;
constexpr int CHUNK_SMALL_MAX = 65536;
constexpr int DNT = 256;           // threads per CTA
constexpr int DWARPS = DNT / 32;

__host__ __device__ constexpr int chunk_of(int N) {
  return N <= CHUNK_SMALL_MAX ? CHUNK_SMALL : CHUNK;
}

// Per-warp per-expert counts of this CTA's slice.  The warp's ids are read
// once, all loads in flight together, into eid (-1: no assignment, or an id
// outside [0,E), which is reported and skipped).  wc: [DWARPS][E] in shared
// memory.
template <int CH, int ROUNDS = CH / DWARPS / 32>
__device__ __forceinline__ void warp_counts(const int32_t* ids, int N, int E, int base,
                                            int (&eid)[ROUNDS], int* wc, int32_t* status) {
  constexpr int PER_WARP = CH / DWARPS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < DWARPS * E; i += DNT) wc[i] = 0;
  moe::grid_dep_wait();
  const int w0 = base + warp * PER_WARP;
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    const int f = w0 + 32 * i + lane;
    eid[i] = f < N ? moe::ld_prod(ids + f) : -1;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    int e = eid[i];
    if (w0 + 32 * i + lane < N && (e < 0 || e >= E)) {
      if (status) moe::report(status, MOE_ERR_BAD_INDEX);
      e = -1;
    }
    eid[i] = e;
    const unsigned valid = __ballot_sync(0xffffffffu, e >= 0);
    // Lanes without a valid id get a unique key so they never match.
    const int key = e >= 0 ? e : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * E + e] += __popc(peers & valid);
  }
  __syncthreads();
}

template <int CH>
__global__ void __launch_bounds__(DNT) dispatch_count_kernel(const int32_t* ids,
                                                             int N, int E,
                                                             int32_t* __restrict__ bc,
                                                             int32_t* status) {
  extern __shared__ int wc[];
  int eid[CH / DWARPS / 32];
  warp_counts<CH>(ids, N, E, blockIdx.x * CH, eid, wc, status);
  for (int e = threadIdx.x; e < E; e += DNT) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < DWARPS; ++w) s += wc[w * E + e];
    bc[static_cast<size_t>(blockIdx.x) * E + e] = s;
  }
  moe::grid_dep_launch();
}

// Exclusive prefix of v over the 256 threads of the CTA (a shuffle scan in
// each warp, then the warp totals); *total gets the sum.  tmp: shared [8].
__device__ __forceinline__ int cta_excl_scan(int v, int* tmp, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int ww = 0; ww < DNT / 32; ++ww) {
    const int t = tmp[ww];
    if (ww < warp) before += t;
    all += t;
  }
  __syncthreads();                 // tmp may be reused
  *total = all;
  return before + incl - v;
}

template <int CH>
__global__ void __launch_bounds__(DNT) dispatch_scatter_kernel(
    const int32_t* ids, const float* w, int N, int E, int k,
    const int32_t* bc, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
    int32_t* __restrict__ packed_tok, float* __restrict__ packed_w, int32_t* status) {
  extern __shared__ int wc[];  // [DWARPS][E] counts, then bases
  // The CTA's assignments in local expert-major order (position, f, weight),
  // copied out after the scatter: consecutive local entries of one expert go
  // to consecutive positions, so the stores come in runs instead of one
  // L2 write per assignment.
  constexpr int PER_WARP = CH / DWARPS, ROUNDS = PER_WARP / 32;
  __shared__ int s_pos[CH], s_f[CH];
  __shared__ float s_w[CH];
  __shared__ int s_shift[moe::kMaxExperts];   // local index - position, per expert
  __shared__ int s_tmp[DNT / 32];
  const int base = blockIdx.x * CH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w0 = base + warp * PER_WARP;
  int eid[ROUNDS];
  warp_counts<CH>(ids, N, E, base, eid, wc, nullptr);
  float wv[ROUNDS];
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    const int f = w0 + 32 * i + lane;
    wv[i] = packed_w != nullptr && f < N ? moe::ld_prod(w + f) : 0.f;
  }
  // Every CTA's count of expert e (the count kernel's table, E <= DNT): the
  // expert's total and the part of the CTAs before this one, 16 loads in
  // flight.  Each CTA scans the totals over the experts itself (the offsets;
  // CTA 0 writes counts and offsets), so no launch sits between the count
  // and scatter kernels.
  const int e = threadIdx.x;
  const int B = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  int etot = 0, before = 0;
  if (e < E) {
    constexpr int BATCH = 16;
    for (int b0 = 0; b0 < B; b0 += BATCH) {
      int c[BATCH];
#pragma unroll
      for (int j = 0; j < BATCH; ++j)
        c[j] = b0 + j < B ? moe::ld_prod(bc + static_cast<size_t>(b0 + j) * E + e) : 0;
#pragma unroll
      for (int j = 0; j < BATCH; ++j) {
        etot += c[j];
        if (b0 + j < b) before += c[j];
      }
    }
  }
  int grand = 0;
  const int eoff = cta_excl_scan(etot, s_tmp, &grand);
  if (b == 0) {
    if (e < E) {
      counts[e] = etot;
      offsets[e] = eoff;
    }
    if (e == 0) offsets[E] = grand;
  }
  // Per-warp global bases, and the CTA's total per expert.
  int total = 0, gbase = 0;
  if (e < E) {
    gbase = eoff + before;
    int run = gbase;
#pragma unroll
    for (int ww = 0; ww < DWARPS; ++ww) {
      const int c = wc[ww * E + e];
      wc[ww * E + e] = run;
      run += c;
    }
    total = run - gbase;
  }
  // Local exclusive scan of the totals over the experts.
  int nvalid = 0;
  const int lexcl = cta_excl_scan(total, s_tmp, &nvalid);
  if (e < E) s_shift[e] = lexcl - gbase;
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    const int f = w0 + 32 * i + lane;
    const int ex = eid[i];
    if (f < N && ex < 0) inv_perm[f] = -1;
    const int key = ex >= 0 ? ex : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (ex >= 0) {
      const int p = wc[warp * E + ex] + __popc(peers & lt);
      inv_perm[f] = p;
      const int q = p + s_shift[ex];
      s_pos[q] = p;
      s_f[q] = f;
      s_w[q] = wv[i];
    }
    __syncwarp();
    if (ex >= 0 && lane == __ffs(peers) - 1) wc[warp * E + ex] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int q = threadIdx.x; q < nvalid; q += DNT) {
    const int p = s_pos[q], f = s_f[q];
    perm[p] = f;
    packed_tok[p] = f / k;
    if (packed_w) packed_w[p] = s_w[q];
  }
  moe::grid_dep_launch();
}

// ------------------------------------------------- single-CTA variant ---

// Up to 2048 assignments.  Above that the multi-CTA kernels are faster even
// with their two extra launches: one SM's match / scatter rounds over 8192
// assignments took 18 us, four CTAs of 2048 take 11 us.
constexpr int SMALL_WARPS = 32;
constexpr int SMALL_PER_WARP = 64;
constexpr int SMALL_N = SMALL_WARPS * SMALL_PER_WARP;   // 2048 assignments

__global__ void __launch_bounds__(SMALL_WARPS * 32) dispatch_small_kernel(
    const int32_t* ids, const float* w, int N, int E, int k,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, int32_t* __restrict__ packed_tok,
    float* __restrict__ packed_w, const uint4* x, int row_vecs,
    uint4* __restrict__ xp, int32_t* status) {
  extern __shared__ int wc[];                  // [SMALL_WARPS][E], then the staging arrays
  __shared__ int s_scan[moe::kMaxExperts];
  for (int i = threadIdx.x; i < SMALL_WARPS * E; i += blockDim.x) wc[i] = 0;
  moe::grid_dep_wait();
  __syncthreads();
  moe::dispatch_cta<SMALL_WARPS, SMALL_PER_WARP / 32>(ids, w, N, E, k, counts, offsets, perm,
                                                      inv_perm, packed_tok, packed_w, x,
                                                      row_vecs, xp, status, wc, s_scan,
                                                      wc + SMALL_WARPS * E);
}

// ------------------------------------------------------------- gather ---

constexpr int GW = 4;      // warps per CTA, each an independent copy engine client
constexpr int GSLOTS = 4;  // rows in flight per warp

// Rows [offsets[lo_e], offsets[hi_e]) of x_packed: every valid row for the
// dispatcher (lo_e = 0, hi_e = E), one rank's experts for an expert range.
__global__ void __launch_bounds__(GW * 32) dispatch_gather_kernel(
    const uint8_t* x, const int32_t* packed_tok,
    const int32_t* offsets, int lo_e, int hi_e, int row_bytes,
    uint8_t* __restrict__ xp, int32_t* status) {
  extern __shared__ __align__(128) uint8_t gsm[];
  __shared__ __align__(8) uint64_t bars[GW][GSLOTS];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) != 0) return;
  uint8_t* ring = gsm + static_cast<size_t>(warp) * GSLOTS * row_bytes;
  for (int s = 0; s < GSLOTS; ++s) moe::mbar_init(moe::smem_addr(&bars[warp][s]), 1);
  moe::fence_barrier_init();
  moe::grid_dep_wait();

  const int row0 = moe::ld_prod(offsets + lo_e);
  const int nrows = moe::ld_prod(offsets + hi_e) - row0;  // valid rows (assignments with a valid id)
  const int stride = gridDim.x * GW;
  const int first = blockIdx.x * GW + warp;
  const int mine = first < nrows ? (nrows - first + stride - 1) / stride : 0;
  auto issue = [&](int i) {
    const int p = row0 + first + i * stride;
    const int s = i % GSLOTS;
    const uint32_t bar = moe::smem_addr(&bars[warp][s]);
    moe::mbar_arrive_expect_tx(bar, row_bytes);
    moe::bulk_g2s(moe::smem_addr(ring + static_cast<size_t>(s) * row_bytes),
                  x + static_cast<size_t>(moe::ld_prod(packed_tok + p)) * row_bytes, row_bytes, bar);
  };
  const int prologue = mine < GSLOTS ? mine : GSLOTS;
  for (int i = 0; i < prologue; ++i) issue(i);
  for (int i = 0; i < mine; ++i) {
    const int s = i % GSLOTS;
    const int p = row0 + first + i * stride;
    if (!moe::mbar_wait(moe::smem_addr(&bars[warp][s]), (i / GSLOTS) & 1)) {
      moe::report(status, MOE_ERR_TIMEOUT);
      // Let every load already issued land before the CTA leaves.
      const int last = mine < i + GSLOTS ? mine : i + GSLOTS;
      for (int j = i + 1; j < last; ++j)
        moe::mbar_wait(moe::smem_addr(&bars[warp][j % GSLOTS]), (j / GSLOTS) & 1);
      break;
    }
    moe::bulk_s2g(xp + static_cast<size_t>(p) * row_bytes,
                  moe::smem_addr(ring + static_cast<size_t>(s) * row_bytes), row_bytes);
    moe::bulk_commit();
    if (i + GSLOTS < mine) {
      moe::bulk_wait_read_all();   // this slot's store has read its bytes
      issue(i + GSLOTS);
    }
  }
  moe::bulk_wait_all();
  moe::grid_dep_launch();
}

// Rows too large for the shared-memory ring: one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) dispatch_gather_vec_kernel(
    const uint4* x, const int32_t* packed_tok,
    const int32_t* offsets, int lo_e, int hi_e, int row_vecs,
    uint4* __restrict__ xp) {
  moe::grid_dep_wait();
  const int row_end = moe::ld_prod(offsets + hi_e);
  const int lane = threadIdx.x & 31;
  for (int p = moe::ld_prod(offsets + lo_e) + ((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
       p < row_end; p += (gridDim.x * blockDim.x) >> 5) {
    const uint4* src = x + static_cast<size_t>(moe::ld_prod(packed_tok + p)) * row_vecs;
    uint4* dst = xp + static_cast<size_t>(p) * row_vecs;
    for (int v0 = lane; v0 < row_vecs; v0 += 32 * 8) {
      uint4 q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + 32 * j < row_vecs) q[j] = moe::ld_prod(src + v0 + 32 * j);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + 32 * j < row_vecs) dst[v0 + 32 * j] = q[j];
    }
  }
  moe::grid_dep_launch();
}

}  // namespace

namespace moe_host {

size_t dispatch_ws_bytes(int T, int k, int E) {
  const size_t N = static_cast<size_t>(T) * k;
  const size_t ch = N <= static_cast<size_t>(CHUNK_SMALL_MAX) ? CHUNK_SMALL : CHUNK;
  const size_t B = (N + ch - 1) / ch;
  return std::max<size_t>(B * E * sizeof(int32_t), 256);
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_dispatch(const int32_t* ids, const float* w, const void* x, int T, int H,
                            int E, int k, int dtype, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv_perm, int32_t* packed_tok,
                            float* packed_w, void* x_packed, void* ws, int32_t* status,
                            cudaStream_t s) {
  const int N = T * k;
  const int es = dtype == MOE_BF16 ? 2 : 4;
  const int row_bytes = H * es;
  if (N <= SMALL_N) {
    // One CTA copies at most 128 KiB of rows; more goes to the multi-CTA gather.
    const bool fuse_gather =
        x != nullptr && static_cast<size_t>(N) * row_bytes <= (static_cast<size_t>(128) << 10);
    // per-warp counts, then perm, packed_tok and packed_w staged (at most 128 KiB)
    const size_t sm = sizeof(int) * (static_cast<size_t>(SMALL_WARPS) * E + 3 * SMALL_N);
    cudaError_t err =
        ensure_smem(reinterpret_cast<const void*>(dispatch_small_kernel), static_cast<int>(sm));
    if (err != cudaSuccess) return err;
    err = launch_pdl(
        dispatch_small_kernel, dim3(1), dim3(SMALL_WARPS * 32), sm, s,
        0, ids, w, N, E, k, counts, offsets, perm, inv_perm, packed_tok, w ? packed_w : nullptr,
        fuse_gather ? static_cast<const uint4*>(x) : nullptr, row_bytes / 16,
        static_cast<uint4*>(x_packed), status);
    if (err != cudaSuccess || x == nullptr || fuse_gather) return err;
  } else {
    const bool small = chunk_of(N) == CHUNK_SMALL;
    const int ch = chunk_of(N);
    const int B = (N + ch - 1) / ch;
    int32_t* bc = static_cast<int32_t*>(ws);
    const size_t wsm = sizeof(int) * DWARPS * E;
    cudaError_t err =
        small ? launch_pdl(dispatch_count_kernel<CHUNK_SMALL>, dim3(B), dim3(DNT), wsm, s, 0,
                           ids, N, E, bc, status)
              : launch_pdl(dispatch_count_kernel<CHUNK>, dim3(B), dim3(DNT), wsm, s, 0, ids, N,
                           E, bc, status);
    if (err == cudaSuccess)
      err = small ? launch_pdl(dispatch_scatter_kernel<CHUNK_SMALL>, dim3(B), dim3(DNT), wsm, s,
                               0, ids, w, N, E, k, static_cast<const int32_t*>(bc), counts,
                               offsets, perm, inv_perm, packed_tok, w ? packed_w : nullptr,
                               status)
                  : launch_pdl(dispatch_scatter_kernel<CHUNK>, dim3(B), dim3(DNT), wsm, s, 0,
                               ids, w, N, E, k, static_cast<const int32_t*>(bc), counts, offsets,
                               perm, inv_perm, packed_tok, w ? packed_w : nullptr, status);
    if (err != cudaSuccess || x == nullptr) return err;
  }
  return launch_gather(x, packed_tok, offsets, 0, E, N, H, dtype, x_packed, status, s);
}

cudaError_t launch_gather(const void* x, const int32_t* packed_tok, const int32_t* offsets,
                          int lo_e, int hi_e, int N, int H, int dtype, void* x_packed,
                          int32_t* status, cudaStream_t s) {
  const int es = dtype == MOE_BF16 ? 2 : 4;
  const int row_bytes = H * es;
  const size_t gsm = static_cast<size_t>(GW) * GSLOTS * row_bytes;
  if (gsm > 200 * 1024) {
    const int grid = std::max(1, std::min((N + 7) / 8, num_sms() * 8));
    return launch_pdl(dispatch_gather_vec_kernel, dim3(grid), dim3(256), 0, s, 0,
                      static_cast<const uint4*>(x), packed_tok, offsets, lo_e, hi_e,
                      row_bytes / 16, static_cast<uint4*>(x_packed));
  }
  cudaError_t err =
      ensure_smem(reinterpret_cast<const void*>(dispatch_gather_kernel), static_cast<int>(gsm));
  if (err != cudaSuccess) return err;
  const int ctas_per_sm = std::max(1, static_cast<int>((200 * 1024) / gsm));
  const int grid = std::max(1, std::min((N + GW - 1) / GW, num_sms() * ctas_per_sm));
  return launch_pdl(dispatch_gather_kernel, dim3(grid), dim3(GW * 32), gsm, s, 0,
                    static_cast<const uint8_t*>(x), packed_tok, offsets, lo_e, hi_e, row_bytes,
                    static_cast<uint8_t*>(x_packed), status);
}

}  // namespace moe_host

// ----------------------------------------------- allocation-free variant ---
//
// moe_dispatch_noalloc runs the same four kernels as moe_dispatch, but its
// per-CTA count table lives in the fixed array below instead of a
// caller-allocated workspace.  It is for callers that cannot call
// cudaMalloc (or any allocator) at the point where they dispatch: a C host
// program whose device memory is carved up by someone else, a plugin of a
// framework that does not expose its allocator, or a serving loop that
// forbids allocation after start-up.  Every GPU that loads this library
// holds the array (128 KiB) until the process exits.

namespace {
constexpr int kNoAllocScratchInts = 32768;   // 128 KiB: ceil(T*k / 2048) * E entries
constexpr int kMaxDevices = 64;
}  // namespace

static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchInts];

namespace {

// Id of the calling thread's current CUDA context (0 if it cannot be read).
// Context ids are never reused within a process, so a cached address keyed
// on one cannot outlive the context it was taken in (cudaDeviceReset
// destroys the primary context; the next one gets a new id).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_cur == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_dispatch_scratch on the current device.  In host code
// the array's name only stands in for the symbol; the address a kernel may
// use comes from cudaGetSymbolAddress, called with the device current.  It is
// cached per device together with the id of the context it was taken in,
// and looked up again whenever that context has changed (after a
// cudaDeviceReset, say), so a stale address is never handed to a kernel.
cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* cached[kMaxDevices] = {};
  static unsigned long long cached_ctx[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();   // 0 before the first runtime call
  if (cached[dev] == nullptr || ctx == 0 || cached_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);    // makes the primary context current
    if (e != cudaSuccess) return e;
    cached[dev] = p;
    cached_ctx[dev] = current_context_id();
  }
  *out = cached[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int moe_dispatch_noalloc(const int32_t* topk_ids, const float* topk_w, const void* x,
                                    int T, int H, int E, int k, int dtype, int32_t* counts,
                                    int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                    int32_t* packed_tok, float* packed_w, void* x_packed,
                                    int32_t* status, void* stream) {
  moe_host::set_last_error("");
  if (T < 1 || k < 1 || E < 1 || E > moe::kMaxExperts || k > E || k > moe::kMaxTopK) {
    moe_host::set_last_error("moe_dispatch_noalloc: need T >= 1, 1 <= k <= min(E, 8), 1 <= E <= 256");
    return MOE_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(T) * k >= (1ll << 30)) {
    moe_host::set_last_error("moe_dispatch_noalloc: T*k too large");
    return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe_host::dispatch_ws_bytes(T, k, E);
  if (need > sizeof(int32_t) * kNoAllocScratchInts) {
    moe_host::set_last_error(
        "moe_dispatch_noalloc: ceil(T*k/2048)*E = " + std::to_string(need / sizeof(int32_t)) +
        " count entries exceed the fixed scratch of 32768 (128 KiB); use moe_dispatch with a "
        "workspace");
    return MOE_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) {
    moe_host::set_last_error(std::string("moe_dispatch_noalloc: cudaGetSymbolAddress: ") +
                             cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  // The remaining argument checks and the launches are those of moe_dispatch
  // (which sets moe_last_error() itself).
  return moe_dispatch(topk_ids, topk_w, x, T, H, E, k, dtype, counts, offsets, perm, inv_perm,
                      packed_tok, packed_w, x_packed, scratch,
                      sizeof(int32_t) * kNoAllocScratchInts, status, stream);
}
