// Executor, bf16: persistent grouped GEMM on the 5th-generation tensor cores.
//
// DWDP-Triton-MoE-Inference-Engine README, "Executor Module": execute the
// expert modules over expert-major ranges, apply routing weights, write
// packed expert outputs.  Experts are SwiGLU MLPs with the fused gate/up
// buffer w13 [E, 2I, H] (gate w1 rows [0,I), up w3 rows [I,2I): the
// w13_weight layout of modelexpress-client's test_reshard_refit_moe_experts.py)
// and w2 [E, H, I].
//
// Two launches of one kernel template:
//   pass 1 (EPI_SWIGLU): A = x_packed [N,H], B = w13[e];
//                        h[p, f] = silu(gate) * up   (bf16 out)
//   pass 2 (EPI_SCALE):  A = h [N,I],        B = w2[e];
//                        y_packed[p, c] = packed_w[p] * acc  (fp32 out, so the
//                        merger adds the k terms before the one bf16 rounding)
//
// Tile = 128 packed rows (tokens of one expert; MMA M) x 256 weight rows
// (MMA N) x K.  In pass 1 the 256 weight rows are 128 gate rows and the 128
// matching up rows (one 3-D TMA box over [2E, I, H]), so column c and column
// 128 + c of the accumulator are the gate and up value of the same feature
// and the SwiGLU is thread-local.  I is a multiple of 64: when it is not one
// of 128, the last feature tile reaches 64 rows past I, which the box reads
// as zeros and the epilogue does not store.  The tile list is derived on the device from
// `offsets` (the scheduler of the README's "Scheduler Module", folded into
// the kernel): expert e owns ceil(count_e / 128) token tiles x (rows / 256)
// weight tiles, token tiles fastest, so CTAs running at the same time share a
// weight tile through L2.  Experts with no rows own no tiles.
//
// Shared expert (diffulex.moe.layer, "SharedExpertMLP").  With SHARED the
// same launches also run a second group: every row of its own input x [T,H]
// through its own w13s [2Is,H] (pass 1, into h_s) and w2s [H,Is] (pass 2,
// into y_s, no routing weight).  Its tiles are numbered before the routed
// ones, so the two weight streams share the SMs instead of following each
// other.  The routed-only build (SHARED = false) carries none of it.
//
// Split-K.  When a pass has fewer tiles than two per CTA (decode batches, a
// shared expert, a long K), every CTA derives the same split count S from the
// tile count, the grid and K, and the work unit becomes (tile, K-slice).  A
// shared group whose K is longer than the routed one is cut into more slices,
// about as long as the routed units.  A unit stores the valid rows of its fp32
// partial in the workspace slot numbered like the unit; the last unit of a
// tile to finish (a per-tile arrival counter) adds the S partials in slice
// order (deterministic) and applies the epilogue.  The counter returns to zero
// for the next call.
//
// Scheduling.  CTA b starts with unit b.  With a workspace, later units are
// handed out dynamically: the producer warp takes the next unit from a
// global ticket counter and passes its id to the MMA and epilogue warps
// through a small shared-memory ring, so a CTA whose units run fast takes more
// of them; the last CTA to exit resets the ticket for the next launch.
// Without one, CTA b takes units b, b+grid, b+2*grid, ...
//
// Waits.  The waits of the main loops (unit ring, stage ring, accumulators)
// are bounded by `wait_ns` (normally the 2 s budget; a test hook shortens it
// so that ordinary waits run out and the abort path runs).  The drain waits
// at the end -- every issued copy landed, every issued MMA completed -- always
// keep the full budget, so nothing is in flight when the CTA leaves.
//
// CTA = 6 warps, one CTA per SM, persistent over units:
//   warp 0    TMA producer   (4-stage ring, 48 KB per stage, 128B swizzle;
//                             5 stages of 36 KB when no tile has over 32 rows)
//   warp 1    MMA issuer     (tcgen05.mma kind::f16, M128 N256 K16; owns TMEM)
//   warps 2-5 epilogue       (tcgen05.ld from the TMEM accumulator, math, store)
// The two 256-column fp32 accumulators are double-buffered in TMEM, so the
// epilogue of one unit overlaps the MMAs of the next.  Every wait is bounded;
// a wait that runs out reports MOE_ERR_TIMEOUT, the CTA drains what it issued
// and frees its TMEM.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int B_BYTES = BN * BK * 2;
constexpr int MAX_STAGES = 5;
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = moe::idesc_bf16_f32(BM, BN);
constexpr int MAX_SPLITS = 16;
constexpr int COUNTER_INTS = 4096;                        // per-tile arrival counters, then
constexpr int SCHED_TICKET = COUNTER_INTS - 2;            // the unit ticket and the
constexpr int SCHED_DONE = COUNTER_INTS - 1;              // CTA exit count of dynamic scheduling
constexpr int UNIT_RING = 8;                              // unit ids handed from producer to consumers
constexpr size_t PARTIAL_BYTES = sizeof(float) * BM * BN;  // one unit's partial slot

enum { EPI_SWIGLU = 0, EPI_SCALE = 1 };

struct Ctl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t ufull[UNIT_RING];    // producer -> MMA + epilogue: unit id published
  uint64_t uempty[UNIT_RING];   // MMA + 4 epilogue warps -> producer: slot read
  int uid[UNIT_RING];
  uint32_t tmem_base;
  int abort;
  int splits;          // S: K-slices per routed tile (1 = no split)
  int splits2;         // K-slices per shared-expert tile
  int last_flag;       // epilogue: this unit is the last of its tile
  int slot_rows;       // rows of one split-K partial slot (the fullest tile's valid rows)
  int n2;              // tiles of the second group (a shared expert), numbered first
  int mte2;            // its token tiles
  int rows2;           // its rows
  int offs[moe::kMaxExperts + 1];
  int tstart[moe::kMaxExperts + 1];   // first tile of routed expert e (after the n2 shared tiles)
};

constexpr int STAGE_OUT_BYTES = BM * 128;                  // epilogue staging: 128 rows x 128 B
// The staging buffer starts on a 1024-byte boundary: TMA stores read it with
// the 128-byte swizzle, whose pattern is anchored there.
constexpr size_t CTL_BYTES = (sizeof(Ctl) + 1023) / 1024 * 1024;
// The stage ring.  A stage holds the A tile (AR rows of activations) and
// then the B tile (256 weight rows), each 64 columns wide.  AR = 128 in
// general; AR = 32 when no tile has more than 32 rows (decode batches): the
// MMA still reads 128 rows of A, the 96 beyond the loaded ones falling inside
// the same stage's B tile -- garbage in accumulator rows that are never
// stored -- and the 12 KB saved per stage buy a fifth stage, 25 % more weight
// bytes in flight per SM.
//
// A routed tile with at most 32 (64) valid rows loads only 32 (64) rows of
// A, in one box; the rows not loaded hold stale data of an earlier stage and
// likewise only reach accumulator rows that are never stored.  A-tile
// reads, although they hit L2, slow the weight stream from DRAM (a TMA-only
// probe of the builder's w13 shape: 6.38 TB/s of weights alone, 5.07 with a
// 16 KB A box per 32 KB weight box, 5.97 with a 4 KB one).  One box per
// stage matters as much: four 32-row boxes instead of one 128-row box made
// the prefill GEMMs 10-15 % slower.
template <int AR>
struct Ring {
  static constexpr int A_B = AR * BK * 2;
  static constexpr int ST_B = A_B + B_BYTES;
  static constexpr int N = AR == BM ? 4 : 5;
  static constexpr size_t SMEM = 1024 + N * ST_B + CTL_BYTES + STAGE_OUT_BYTES;
  static_assert(AR == BM || (AR >= 8 && AR % 8 == 0 && A_B + B_BYTES >= BM * BK * 2),
                "a short A tile must be followed by at least 128 rows' worth of the stage");
  static_assert(N <= MAX_STAGES && SMEM <= 227 * 1024, "stage ring exceeds shared memory");
  static_assert(ST_B % 1024 == 0 && A_B % 1024 == 0, "tiles must stay 1024-byte aligned");
};

// A work unit: tile (group g, expert e, weight tile nt, token tile mt) and
// its K-slice [kb0, kb1).  Group 1 is the optional shared expert (all rows of
// its own input), group 0 the routed experts.  Its rows are [row0, rend).
struct Unit {
  int tile, g, e, nt, mt, ks, S, kb0, kb1, row0, rend;
};

template <bool SHARED>
__device__ __forceinline__ Unit decode_unit(const Ctl& c, int E, int kblocks, int kblocks2,
                                            int u) {
  // Units: the shared tiles' slices first (splits2 each), then the routed
  // tiles' (splits each).  The unit id is also the partial slot of a slice.
  Unit r;
  const int u2 = SHARED ? c.n2 * c.splits2 : 0;
  if (SHARED && u < u2) {
    r.S = c.splits2;
    r.tile = u / r.S;
    r.ks = u - r.tile * r.S;
  } else {
    r.S = c.splits;
    const int n2 = SHARED ? c.n2 : 0;
    const int v = u - u2;
    r.tile = n2 + v / r.S;
    r.ks = v - (r.tile - n2) * r.S;
  }
  int kb;
  if (SHARED && r.tile < c.n2) {
    r.g = 1;
    r.e = 0;
    r.nt = r.tile / c.mte2;
    r.mt = r.tile - r.nt * c.mte2;
    r.row0 = r.mt * BM;
    r.rend = c.rows2;
    kb = kblocks2;
  } else {
    // largest e with tstart[e] <= tile (experts without tiles share their successor's start)
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (c.tstart[mid] <= r.tile) lo = mid; else hi = mid - 1;
    }
    r.g = 0;
    r.e = lo;
    const int mte = (c.offs[r.e + 1] - c.offs[r.e] + BM - 1) / BM;
    const int local = r.tile - c.tstart[r.e];
    r.nt = local / mte;
    r.mt = local - r.nt * mte;
    r.row0 = c.offs[r.e] + r.mt * BM;
    r.rend = c.offs[r.e + 1];
    kb = kblocks;
  }
  r.kb0 = (r.ks * kb) / r.S;
  r.kb1 = ((r.ks + 1) * kb) / r.S;
  return r;
}

// Split count: 1 when there are at least two tiles per CTA; otherwise the
// smallest S whose units fill the grid's waves to >= 90% (else the best one),
// with >= 4 K-blocks per unit, the units within the workspace's partial slots
// (max_units), and at most 128 partial rows per tile (S x the fullest tile's
// valid rows), since one CTA reads them all back.
__device__ int choose_splits(int tiles, int grid, int kblocks, int max_units, int rows_max) {
  if (tiles <= 0 || tiles >= 2 * grid) return 1;
  int smax = min(MAX_SPLITS, kblocks / 4);
  smax = min(smax, max_units / tiles);
  smax = min(smax, max(2, BM / max(1, rows_max)));
  if (smax <= 1) return 1;
  int best = 1;
  float best_eff = 0.f;
  for (int s = 1; s <= smax; ++s) {
    const int units = tiles * s;
    const int waves = (units + grid - 1) / grid;
    const float eff = static_cast<float>(units) / static_cast<float>(waves * grid);
    if (eff >= 0.9f) return s;
    if (eff > best_eff + 1e-6f) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

__device__ __forceinline__ void set_abort(Ctl& c, int32_t* status) {
  moe::report(status, MOE_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c.abort) = 1;
}

__device__ __forceinline__ bool aborted(const Ctl& c) {
  return *reinterpret_cast<const volatile int*>(&c.abort) != 0;
}

__device__ __forceinline__ void epi_bar() {   // the 4 epilogue warps only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + __expf(-g)) * u; }

// Direct per-thread row stores, used when a tile has few valid rows (there
// the staging barriers cost more than the scattered stores they save).
__device__ __forceinline__ void store_f32x32(float* dst, const uint32_t* a, const uint32_t* b,
                                             float sc) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    d4[j] = make_float4(__uint_as_float(a[4 * j]) * sc, __uint_as_float(a[4 * j + 1]) * sc,
                        __uint_as_float(a[4 * j + 2]) * sc, __uint_as_float(a[4 * j + 3]) * sc);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    d4[4 + j] = make_float4(__uint_as_float(b[4 * j]) * sc, __uint_as_float(b[4 * j + 1]) * sc,
                            __uint_as_float(b[4 * j + 2]) * sc, __uint_as_float(b[4 * j + 3]) * sc);
}

constexpr int STAGE_MIN_ROWS = 32;   // stage the epilogue only above this many valid rows

// Epilogue staging.  A thread owns one tile row (its TMEM lane); rows are
// written to global memory through a 128 row x 128 byte shared buffer so that
// each warp store covers whole 128-byte row segments (4 rows per instruction)
// instead of 32 scattered 16-byte pieces.  16-byte chunk j of row r sits at
// position j ^ (r & 7): conflict-free both when 32 lanes each write their own
// row and when 8 lanes read one row.
__device__ __forceinline__ void stage_put(uint8_t* stg, int row, int j, uint4 v) {
  reinterpret_cast<uint4*>(stg + row * 128)[j ^ (row & 7)] = v;
}

// Write rows [0, nvalid) of the staged 128-byte chunk to gtile + r * ld_bytes;
// warp quarter wq handles rows 32*wq .. 32*wq + 31.
__device__ __forceinline__ void stage_flush(const uint8_t* stg, int wq, int lane, int nvalid,
                                            uint8_t* gtile, size_t ld_bytes) {
  const int j = lane & 7;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = wq * 32 + it * 4 + (lane >> 3);
    if (r < nvalid) {
      const uint4 v = reinterpret_cast<const uint4*>(stg + r * 128)[j ^ (r & 7)];
      *reinterpret_cast<uint4*>(gtile + static_cast<size_t>(r) * ld_bytes + j * 16) = v;
    }
  }
}

// 32 fp32 accumulator columns (two TMEM loads) scaled by sc -> 8 staged chunks.
__device__ __forceinline__ void stage_f32x32(uint8_t* stg, int row, const uint32_t* a,
                                             const uint32_t* b, float sc) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    stage_put(stg, row, j,
              make_uint4(__float_as_uint(__uint_as_float(a[4 * j]) * sc),
                         __float_as_uint(__uint_as_float(a[4 * j + 1]) * sc),
                         __float_as_uint(__uint_as_float(a[4 * j + 2]) * sc),
                         __float_as_uint(__uint_as_float(a[4 * j + 3]) * sc)));
#pragma unroll
  for (int j = 0; j < 4; ++j)
    stage_put(stg, row, 4 + j,
              make_uint4(__float_as_uint(__uint_as_float(b[4 * j]) * sc),
                         __float_as_uint(__uint_as_float(b[4 * j + 1]) * sc),
                         __float_as_uint(__uint_as_float(b[4 * j + 2]) * sc),
                         __float_as_uint(__uint_as_float(b[4 * j + 3]) * sc)));
}

// 64 fp32 accumulator columns (four TMEM loads) scaled by sc and rounded to
// fp16 -> 8 staged chunks (128 bytes of the row).  Returns the largest
// magnitude stored (for the fp16 range check).
__device__ __forceinline__ uint4 h16x8(const uint32_t* a, float sc, float& mx) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = __uint_as_float(a[i]) * sc;
    mx = fmaxf(mx, fabsf(v[i]));
  }
  return make_uint4(moe::pack_f16x2(v[0], v[1]), moe::pack_f16x2(v[2], v[3]),
                    moe::pack_f16x2(v[4], v[5]), moe::pack_f16x2(v[6], v[7]));
}

__device__ __forceinline__ float stage_h16x64(uint8_t* stg, int row, const uint32_t (&a)[4][16],
                                              float sc) {
  float mx = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int j = 0; j < 2; ++j) stage_put(stg, row, 2 * q + j, h16x8(&a[q][8 * j], sc, mx));
  return mx;
}

// The same 64 columns stored directly to one fp16 row (dst: 16-byte aligned).
__device__ __forceinline__ float store_h16x64(__half* dst, const uint32_t (&a)[4][16], float sc) {
  float mx = 0.f;
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int j = 0; j < 2; ++j) d4[2 * q + j] = h16x8(&a[q][8 * j], sc, mx);
  return mx;
}

// YH (pass 2 only): y_packed and the shared expert's y are fp16 -- each
// element rounded once, after the fp32 accumulation and the routing-weight
// scale -- instead of fp32.  A magnitude above the fp16 range is reported
// (MOE_ERR_OVERFLOW); the element becomes inf.
template <int EPI, bool SHARED, bool YH, int AR>
__global__ void __launch_bounds__(NTHREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA64,
                        const __grid_constant__ CUtensorMap tmA32,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmB2,
                        const __grid_constant__ CUtensorMap tmY,
                        const __grid_constant__ CUtensorMap tmY2,
                        const int32_t* __restrict__ offsets, int E, int K, int ntw,
                        int rows_per_expert, const float* packed_w,
                        void* __restrict__ out, int ldo, int rows2, int K2, int ntw2,
                        void* __restrict__ out2, int ldo2, int* __restrict__ counters,
                        float* __restrict__ partials, int max_units, int32_t* status,
                        uint64_t wait_ns) {
  using RG = Ring<AR>;
  constexpr int STAGES = RG::N;
  constexpr int A_BYTES = RG::A_B;
  constexpr int STAGE_BYTES = RG::ST_B;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctl& c = *reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  uint8_t* stg = smem + STAGES * STAGE_BYTES + CTL_BYTES;   // epilogue staging
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kblocks = K / BK;
  const int kblocks2 = K2 / BK;
  rows2 = SHARED ? rows2 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      moe::mbar_init(moe::smem_addr(&c.full[s]), 1);
      moe::mbar_init(moe::smem_addr(&c.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      moe::mbar_init(moe::smem_addr(&c.tfull[b]), 1);
      moe::mbar_init(moe::smem_addr(&c.tempty[b]), 4);
    }
    moe::mbar_init(moe::smem_addr(&c.drain), 1);
    for (int r = 0; r < UNIT_RING; ++r) {
      moe::mbar_init(moe::smem_addr(&c.ufull[r]), 1);
      moe::mbar_init(moe::smem_addr(&c.uempty[r]), 5);
    }
    c.abort = 0;
    moe::fence_barrier_init();
    moe::prefetch_tmap(&tmA);
    if (AR == BM) {
      moe::prefetch_tmap(&tmA64);
      moe::prefetch_tmap(&tmA32);
    }
    moe::prefetch_tmap(&tmB);
    if (rows2 > 0) {
      moe::prefetch_tmap(&tmA2);
      moe::prefetch_tmap(&tmB2);
    }
  }
  if (warp == 1) {
    moe::tmem_alloc(moe::smem_addr(&c.tmem_base), TMEM_COLS);
    moe::tmem_relinquish();
  }
  // Pass 1 reads offsets and x_packed, both written by the kernels just before
  // it, so it waits for them first.  Pass 2's inputs other than h are older:
  // its offsets were final before pass 1 could start (pass 1 waited for them,
  // and pass 2 starts only once every pass-1 CTA has passed that wait), and
  // the weights are constant.  So pass 2 builds its tile table and requests
  // the weights of its first unit while pass 1 still finishes, and waits only
  // before its first read of h.
  constexpr bool EARLY = EPI == EPI_SCALE;
  if (!EARLY) moe::grid_dep_wait();
  if (warp == 2) {
    // Tile table: per-expert token-tile counts, exclusive scan, x ntw.
    // Lane l owns experts [8l, 8l+8); lane 31 also writes the end entries.
    int cnt[8];
    int local = 0;
    int rmax = 0;                     // valid rows of the fullest tile
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      int m = 0;
      if (e < E) {
        // read at L2, the point of coherence (pass 2 reads before its wait)
        const int o0 = __ldcg(offsets + e), o1 = __ldcg(offsets + e + 1);
        c.offs[e] = o0;
        const int rows = o1 - o0;
        m = (rows + BM - 1) / BM;
        rmax = max(rmax, min(rows, BM));
      }
      cnt[j] = m;
      local += m;
    }
    rmax = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(rmax)));
    const int mte2 = (rows2 + BM - 1) / BM;      // the shared group's tiles come first
    const int n2 = mte2 * ntw2;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) c.tstart[e] = n2 + run * ntw;
      run += cnt[j];
    }
    if (lane == 31) {
      c.offs[E] = __ldcg(offsets + E);
      const int tiles = n2 + incl * ntw;
      c.tstart[E] = tiles;
      c.n2 = n2;
      c.mte2 = mte2;
      c.rows2 = rows2;
      const int rt = incl * ntw;                  // routed tiles
      // A partial slot holds only the rows a tile can have (the fullest
      // tile's, rounded up to 8), so decode batches, whose tiles have a row
      // or two, fit many more slots in the workspace and can split finer.
      const int slot_rows = min(BM, max(8, (max(rmax, min(rows2, BM)) + 7) / 8 * 8));
      const int units_cap = static_cast<int>(
          min(static_cast<long long>(max_units) * BM / slot_rows, 1ll << 30));
      int sp = 1, sp2 = 1;
      if (counters != nullptr && partials != nullptr && tiles <= SCHED_TICKET) {
        if (rt == 0) {
          sp2 = choose_splits(n2, gridDim.x, kblocks2, units_cap, min(rows2, BM));
        } else {
          sp = choose_splits(tiles, gridDim.x, kblocks, units_cap, max(rmax, min(rows2, BM)));
          if (n2 > 0 && kblocks2 > kblocks) {
            // a longer shared K is cut into slices about as long as the routed units
            sp2 = min(sp * ((kblocks2 + kblocks - 1) / kblocks), MAX_SPLITS);
            sp2 = min(sp2, max(1, kblocks2 / 4));
            sp2 = min(sp2, max(2, BM / max(1, min(rows2, BM))));
            if (n2 * sp2 + rt * sp > units_cap) sp2 = sp;
          } else {
            sp2 = sp;
          }
        }
      }
      c.splits = sp;
      c.splits2 = sp2;
      c.slot_rows = slot_rows;
    }
  }
  moe::tc_fence_before();
  __syncthreads();
  moe::tc_fence_after();

  const int total = c.n2 * c.splits2 + (c.tstart[E] - c.n2) * c.splits;   // units
  const uint32_t tmem = c.tmem_base;

  // The B operand (weights) of k-block kb of unit un into stage buffer sa,
  // completing on barrier fb.
  // The A box of a unit (its map and rows): 32 or 64 rows for a routed
  // tile with at most that many valid rows, else the full AR rows.
  auto a_rows = [&](const Unit& un) {
    if (AR != BM || (SHARED && un.g)) return AR;
    const int rows = un.rend - un.row0;
    return rows <= 32 ? 32 : (rows <= 64 ? 64 : BM);
  };
  auto a_map = [&](const Unit& un, int ar) -> const CUtensorMap* {
    if (SHARED && un.g) return &tmA2;
    return ar == 32 && AR == BM ? &tmA32 : (ar == 64 ? &tmA64 : &tmA);
  };
  auto stage_tx = [&](int ar) {
    return static_cast<uint32_t>(STAGE_BYTES - A_BYTES + ar * BK * 2);
  };

  auto load_b = [&](const Unit& un, int kb, uint32_t sa, uint32_t fb) {
    if (SHARED && un.g) {
      if (EPI == EPI_SWIGLU)
        moe::tma_load_3d(sa + A_BYTES, &tmB2, fb, kb * BK, un.nt * (BN / 2), 0);
      else
        moe::tma_load_2d(sa + A_BYTES, &tmB2, fb, kb * BK, un.nt * BN);
    } else if (EPI == EPI_SWIGLU) {
      moe::tma_load_3d(sa + A_BYTES, &tmB, fb, kb * BK, un.nt * (BN / 2), 2 * un.e);
    } else {
      moe::tma_load_2d(sa + A_BYTES, &tmB, fb, kb * BK, un.e * rows_per_expert + un.nt * BN);
    }
  };

  // The same k-block of the B operand, requested into L2 only.
  auto prefetch_b = [&](const Unit& un, int kb) {
    if (SHARED && un.g) {
      if (EPI == EPI_SWIGLU)
        moe::tma_prefetch_3d(&tmB2, kb * BK, un.nt * (BN / 2), 0);
      else
        moe::tma_prefetch_2d(&tmB2, kb * BK, un.nt * BN);
    } else if (EPI == EPI_SWIGLU) {
      moe::tma_prefetch_3d(&tmB, kb * BK, un.nt * (BN / 2), 2 * un.e);
    } else {
      moe::tma_prefetch_2d(&tmB, kb * BK, un.e * rows_per_expert + un.nt * BN);
    }
  };

  // Pass 2, before waiting for pass 1: the weights of this CTA's first unit
  // (static: unit blockIdx.x) into the first stages, and the next k-blocks
  // into L2.  Each such stage's barrier expects the whole stage; the A half
  // follows after the wait.
  int pre = 0;                                   // stages whose B half is on its way
  int pre_issued[STAGES] = {};
  if (EARLY && warp == 0 && lane == 0 && static_cast<int>(blockIdx.x) < total) {
    const Unit un = decode_unit<SHARED>(c, E, kblocks, kblocks2, blockIdx.x);
    pre = min(STAGES, un.kb1 - un.kb0);
    const uint32_t tx = stage_tx(a_rows(un));
    for (int s = 0; s < pre; ++s) {
      const uint32_t fb = moe::smem_addr(&c.full[s]);
      moe::mbar_arrive_expect_tx(fb, tx);
      load_b(un, un.kb0 + s, moe::smem_addr(smem + s * STAGE_BYTES), fb);
      pre_issued[s] = 1;
    }
    const int l2_end = min(un.kb1, un.kb0 + pre + 8);
    for (int kb = un.kb0 + pre; kb < l2_end; ++kb) prefetch_b(un, kb);
  }
  if (EARLY) moe::grid_dep_wait();               // h comes from pass 1

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer ---
      int stage = 0;
      uint32_t phase = 0;
      int issued[STAGES] = {};
      for (int s = 0; s < STAGES; ++s) issued[s] = pre_issued[s];
      int uslot = 0;
      uint32_t uphase = 0;
      int next_static = blockIdx.x;
      int npre = pre;                              // the first unit's prefetched k-blocks
      for (;;) {
        // Take the next unit and publish its id (-1: no more work) to the consumers.
        if (!moe::mbar_wait(moe::smem_addr(&c.uempty[uslot]), uphase ^ 1, wait_ns)) {
          set_abort(c, status);
          break;
        }
        int u;
        if (next_static == static_cast<int>(blockIdx.x) || counters == nullptr) {
          u = next_static;                    // the first unit of every CTA is static
          next_static += gridDim.x;
        } else {
          u = gridDim.x + atomicAdd(&counters[SCHED_TICKET], 1);
        }
        if (u >= total || aborted(c)) u = -1;
        c.uid[uslot] = u;
        moe::mbar_arrive(moe::smem_addr(&c.ufull[uslot]));
        if (++uslot == UNIT_RING) {
          uslot = 0;
          uphase ^= 1;
        }
        if (u < 0) break;
        const Unit un = decode_unit<SHARED>(c, E, kblocks, kblocks2, u);
        const int arow = un.row0;
        const bool g1 = SHARED && un.g;
        const int ar = a_rows(un);
        const CUtensorMap* ma = a_map(un, ar);
        const uint32_t tx = stage_tx(ar);
        bool ok = true;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          const uint32_t fb = moe::smem_addr(&c.full[stage]);
          const uint32_t sa = moe::smem_addr(smem + stage * STAGE_BYTES);
          if (kb - un.kb0 < npre) {
            // B already requested before the wait (fresh stage, nothing to wait for)
            moe::tma_load_2d(sa, ma, fb, kb * BK, arow);
          } else {
            if (!moe::mbar_wait(moe::smem_addr(&c.empty[stage]), phase ^ 1, wait_ns)) {
              set_abort(c, status);
              ok = false;
              break;
            }
            moe::mbar_arrive_expect_tx(fb, tx);
            moe::tma_load_2d(sa, ma, fb, kb * BK, arow);
            load_b(un, kb, sa, fb);
            ++issued[stage];
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        npre = 0;
        if (!ok) break;
      }
      // Drain: every load issued has landed before the CTA can leave.
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > 0) moe::mbar_wait(moe::smem_addr(&c.full[s]), (issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA ---
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      int uslot = 0;
      uint32_t uphase = 0;
      for (;; ++i) {
        if (!moe::mbar_wait(moe::smem_addr(&c.ufull[uslot]), uphase, wait_ns)) {
          set_abort(c, status);
          break;
        }
        const int u = c.uid[uslot];
        moe::mbar_arrive(moe::smem_addr(&c.uempty[uslot]));
        if (++uslot == UNIT_RING) {
          uslot = 0;
          uphase ^= 1;
        }
        if (u < 0) break;
        const Unit un = decode_unit<SHARED>(c, E, kblocks, kblocks2, u);
        const int buf = i & 1;
        if (!moe::mbar_wait(moe::smem_addr(&c.tempty[buf]), ((i >> 1) & 1) ^ 1, wait_ns)) {
          set_abort(c, status);
          break;
        }
        moe::tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
        bool ok = true;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          if (!moe::mbar_wait(moe::smem_addr(&c.full[stage]), phase, wait_ns)) {
            set_abort(c, status);
            ok = false;
            break;
          }
          moe::tc_fence_after();
          const uint32_t sa = moe::smem_addr(smem + stage * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = moe::sw128_kmajor_desc(sa + kk * 32);
            const uint64_t bd = moe::sw128_kmajor_desc(sa + A_BYTES + kk * 32);
            moe::tc_mma_f16(d, ad, bd, IDESC, (kb > un.kb0 || kk > 0) ? 1u : 0u);
          }
          moe::tc_commit(moe::smem_addr(&c.empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        moe::tc_commit(moe::smem_addr(&c.tfull[buf]));
      }
      // Drain: all MMAs this thread issued have completed.
      moe::tc_commit(moe::smem_addr(&c.drain));
      moe::mbar_wait(moe::smem_addr(&c.drain), 0);
    }
  } else {
    // ------------------------------------------------------- epilogue ---
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;          // row of the tile owned by this thread
    int i = 0;
    int uslot = 0;
    uint32_t uphase = 0;
    for (;; ++i) {
      if (!moe::mbar_wait(moe::smem_addr(&c.ufull[uslot]), uphase, wait_ns)) {
        set_abort(c, status);
        break;
      }
      const int u = c.uid[uslot];
      __syncwarp();
      if (lane == 0) moe::mbar_arrive(moe::smem_addr(&c.uempty[uslot]));
      if (++uslot == UNIT_RING) {
        uslot = 0;
        uphase ^= 1;
      }
      if (u < 0) break;
      const int buf = i & 1;
      if (!moe::mbar_wait(moe::smem_addr(&c.tfull[buf]), (i >> 1) & 1, wait_ns)) {
        set_abort(c, status);
        break;
      }
      moe::tc_fence_after();
      const Unit un = decode_unit<SHARED>(c, E, kblocks, kblocks2, u);
      const int rows_valid = un.rend - un.row0;
      const bool live = row < rows_valid;
      const size_t grow = static_cast<size_t>(un.row0 + row);
      const bool g1 = SHARED && un.g;
      void* const uout = g1 ? out2 : out;            // the unit's group's output
      const int uldo = g1 ? ldo2 : ldo;
      const float* const upw = g1 ? nullptr : packed_w;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(buf * BN);
      const int nvalid = rows_valid < BM ? rows_valid : BM;
      // h columns of this feature tile that exist (pass 1: 64 or 128)
      const int ncol = min(BN / 2, uldo - un.nt * (BN / 2));
      const bool staged = nvalid > STAGE_MIN_ROWS;    // same for all four epilogue warps
      const size_t row0 = static_cast<size_t>(un.row0);
      const int S = un.S;
      if (S == 1) {
        if (EPI == EPI_SWIGLU && !staged) {
          // few valid rows: 16 h columns per step, each thread stores its own row
          __nv_bfloat16* dst =
              static_cast<__nv_bfloat16*>(uout) + grow * uldo + un.nt * (BN / 2);
#pragma unroll 1
          for (int cc = 0; cc < ncol; cc += 16) {
            uint32_t g[16], v[16];
            moe::tmem_ld16(taddr + cc, g);
            moe::tmem_ld16(taddr + BN / 2 + cc, v);
            moe::tmem_ld_wait();
            if (live) {
              uint32_t pk[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                pk[j] = moe::pack_bf16x2(
                    silu_mul(__uint_as_float(g[2 * j]), __uint_as_float(v[2 * j])),
                    silu_mul(__uint_as_float(g[2 * j + 1]), __uint_as_float(v[2 * j + 1])));
              uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
              d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        } else if (EPI == EPI_SWIGLU) {
          // 64 h columns per staged chunk: gate cols hc.., up cols 128+hc..
          uint8_t* gtile = static_cast<uint8_t*>(uout) +
                           (row0 * uldo + un.nt * (BN / 2)) * sizeof(__nv_bfloat16);
#pragma unroll 1
          for (int hc = 0; hc < ncol; hc += 64) {        // same count in all four warps
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              const int cc = hc + half * 32;
              uint32_t g0[16], g1[16], v0[16], v1[16];
              moe::tmem_ld16(taddr + cc, g0);
              moe::tmem_ld16(taddr + cc + 16, g1);
              moe::tmem_ld16(taddr + BN / 2 + cc, v0);
              moe::tmem_ld16(taddr + BN / 2 + cc + 16, v1);
              moe::tmem_ld_wait();
              uint32_t pk[16];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                pk[j] = moe::pack_bf16x2(
                    silu_mul(__uint_as_float(g0[2 * j]), __uint_as_float(v0[2 * j])),
                    silu_mul(__uint_as_float(g0[2 * j + 1]), __uint_as_float(v0[2 * j + 1])));
                pk[8 + j] = moe::pack_bf16x2(
                    silu_mul(__uint_as_float(g1[2 * j]), __uint_as_float(v1[2 * j])),
                    silu_mul(__uint_as_float(g1[2 * j + 1]), __uint_as_float(v1[2 * j + 1])));
              }
#pragma unroll
              for (int j = 0; j < 4; ++j)
                stage_put(stg, row, half * 4 + j,
                          make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]));
            }
            epi_bar();
            stage_flush(stg, q, lane, nvalid, gtile + hc * sizeof(__nv_bfloat16),
                        static_cast<size_t>(uldo) * sizeof(__nv_bfloat16));
            epi_bar();
          }
        } else {
          // fp32 output, 32 columns per step.  Each warp works alone on its
          // 32-row quarter: when all 32 rows belong to the unit it stages
          // them (the 128-byte-swizzled layout a TMA store reads) and one lane
          // hands the 32 x 32 block to the TMA engine, so no thread waits on
          // global stores and no barrier spans the warps; a partly valid
          // quarter stores its valid rows directly.
          const float sc = live ? (upw ? moe::ld_prod(upw + grow) : 1.f) : 0.f;
          const int qrows = min(max(nvalid - q * 32, 0), 32);
          const CUtensorMap* ym = g1 ? &tmY2 : &tmY;
          const uint32_t wstg = moe::smem_addr(stg + q * 32 * 128);
          if (YH) {
            // fp16 output, 64 columns (one 128-byte staged row) per step
            __half* yrow = static_cast<__half*>(uout) + grow * uldo + un.nt * BN;
            float mx = 0.f;
#pragma unroll 1
            for (int cc = 0; cc < BN; cc += 64) {
              uint32_t a[4][16];
#pragma unroll
              for (int j = 0; j < 4; ++j) moe::tmem_ld16(taddr + cc + 16 * j, a[j]);
              moe::tmem_ld_wait();
              if (qrows == 32) {
                if (lane == 0) moe::bulk_wait_read_all();   // the last store has read the stage
                __syncwarp();
                mx = fmaxf(mx, stage_h16x64(stg, row, a, sc));
                moe::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  moe::tma_store_2d(ym, wstg, un.nt * BN + cc, static_cast<int>(row0) + q * 32);
                  moe::bulk_commit();
                }
              } else if (live) {
                mx = fmaxf(mx, store_h16x64(yrow + cc, a, sc));
              }
            }
            if (mx > moe::kF16Max) moe::report(status, MOE_ERR_OVERFLOW);
          }
          uint8_t* gtile =
              static_cast<uint8_t*>(uout) + (row0 * uldo + un.nt * BN) * sizeof(float);
#pragma unroll 1
          for (int cc = 0; cc < (YH ? 0 : BN); cc += 32) {
            uint32_t a[16], b[16];
            moe::tmem_ld16(taddr + cc, a);
            moe::tmem_ld16(taddr + cc + 16, b);
            moe::tmem_ld_wait();
            if (qrows == 32) {
              if (lane == 0) moe::bulk_wait_read_all();   // the last store has read the stage
              __syncwarp();
              stage_f32x32(stg, row, a, b, sc);
              moe::fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                moe::tma_store_2d(ym, wstg, un.nt * BN + cc, static_cast<int>(row0) + q * 32);
                moe::bulk_commit();
              }
            } else if (live) {
              store_f32x32(reinterpret_cast<float*>(gtile) + static_cast<size_t>(row) * uldo + cc,
                           a, b, sc);
            }
          }
        }
        moe::tc_fence_before();
        __syncwarp();
        if (lane == 0) moe::mbar_arrive(moe::smem_addr(&c.tempty[buf]));
      } else {
        // Partial of one K-slice: valid rows to this unit's workspace slot.
        // (In the w2 pass a TMA store of an earlier unit may still be reading
        // this warp's quarter of the staging buffer: let it finish first.)
        if (EPI == EPI_SCALE) {
          if (lane == 0) moe::bulk_wait_read_all();
          __syncwarp();
        }
        const size_t slot = static_cast<size_t>(c.slot_rows) * BN;   // floats per slot
        uint8_t* gtile = reinterpret_cast<uint8_t*>(partials + static_cast<size_t>(u) * slot);
#pragma unroll 1
        for (int cc = 0; cc < BN; cc += 32) {
          uint32_t a[16], b[16];
          moe::tmem_ld16(taddr + cc, a);
          moe::tmem_ld16(taddr + cc + 16, b);
          moe::tmem_ld_wait();
          if (staged) {
            stage_f32x32(stg, row, a, b, 1.f);
            epi_bar();
            stage_flush(stg, q, lane, nvalid, gtile + cc * sizeof(float), BN * sizeof(float));
            epi_bar();
          } else if (live) {
            store_f32x32(reinterpret_cast<float*>(gtile) + static_cast<size_t>(row) * BN + cc, a,
                         b, 1.f);
          }
        }
        moe::tc_fence_before();
        __syncwarp();
        if (lane == 0) moe::mbar_arrive(moe::smem_addr(&c.tempty[buf]));   // TMEM free
        __threadfence();
        epi_bar();
        if (warp == 2 && lane == 0) {
          const int old = atomicAdd(&counters[un.tile], 1);
          const int last = old == S - 1;
          if (last) counters[un.tile] = 0;       // ready for the next call
          c.last_flag = last;
        }
        epi_bar();
        const bool last = c.last_flag != 0;
        epi_bar();                               // everyone read the flag before it changes
        if (last) {
          // All 128 epilogue threads reduce the tile: the S partials of every
          // valid row, summed in slice order (loads of one output batched
          // across slices so they are in flight together).
          __threadfence();
          const int et = threadIdx.x - 64;                // 0..127
          const int nrows = nvalid;
          const float* base = partials + static_cast<size_t>(u - un.ks) * slot;
          if (EPI == EPI_SWIGLU) {
            const int cg = et & 31;                       // h columns 4cg .. 4cg+3
            for (int r = et >> 5; r < nrows && cg * 4 < ncol; r += 4) {
              float4 g = make_float4(0.f, 0.f, 0.f, 0.f), v = g;
              const float* pr = base + static_cast<size_t>(r) * BN + cg * 4;
#pragma unroll
              for (int s = 0; s < MAX_SPLITS; ++s) {
                if (s < S) {
                  const float4 a = __ldcg(reinterpret_cast<const float4*>(pr + s * slot));
                  const float4 b =
                      __ldcg(reinterpret_cast<const float4*>(pr + s * slot + BN / 2));
                  g.x += a.x; g.y += a.y; g.z += a.z; g.w += a.w;
                  v.x += b.x; v.y += b.y; v.z += b.z; v.w += b.w;
                }
              }
              uint2 pk;
              pk.x = moe::pack_bf16x2(silu_mul(g.x, v.x), silu_mul(g.y, v.y));
              pk.y = moe::pack_bf16x2(silu_mul(g.z, v.z), silu_mul(g.w, v.w));
              *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(uout) + (row0 + r) * uldo +
                                        un.nt * (BN / 2) + cg * 4) = pk;
            }
          } else {
            const int cg = et & 63;                       // y columns 4cg .. 4cg+3
            for (int r = et >> 6; r < nrows; r += 2) {
              float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
              const float* pr = base + static_cast<size_t>(r) * BN + cg * 4;
#pragma unroll
              for (int s = 0; s < MAX_SPLITS; ++s) {
                if (s < S) {
                  const float4 a = __ldcg(reinterpret_cast<const float4*>(pr + s * slot));
                  v.x += a.x; v.y += a.y; v.z += a.z; v.w += a.w;
                }
              }
              const float sc = upw ? moe::ld_prod(upw + row0 + r) : 1.f;
              if (YH) {
                const float4 o = make_float4(v.x * sc, v.y * sc, v.z * sc, v.w * sc);
                if (fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))) >
                    moe::kF16Max)
                  moe::report(status, MOE_ERR_OVERFLOW);
                uint2 pk;
                pk.x = moe::pack_f16x2(o.x, o.y);
                pk.y = moe::pack_f16x2(o.z, o.w);
                *reinterpret_cast<uint2*>(static_cast<__half*>(uout) + (row0 + r) * uldo +
                                          un.nt * BN + cg * 4) = pk;
              } else {
                *reinterpret_cast<float4*>(static_cast<float*>(uout) + (row0 + r) * uldo +
                                           un.nt * BN + cg * 4) =
                    make_float4(v.x * sc, v.y * sc, v.z * sc, v.w * sc);
              }
            }
          }
        }
      }
    }
  }

  if (EPI == EPI_SCALE && warp >= 2 && lane == 0)
    moe::bulk_wait_all();          // this warp's TMA stores are complete before the grid ends
  moe::grid_dep_launch();
  moe::tc_fence_before();
  __syncthreads();
  moe::tc_fence_after();
  if (warp == 1) moe::tmem_dealloc(tmem, TMEM_COLS);
  if (threadIdx.x == 0 && counters != nullptr) {
    // The last CTA to leave returns the ticket (and the exit count) to zero.
    __threadfence();
    if (atomicAdd(&counters[SCHED_DONE], 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(&counters[SCHED_TICKET], 0);
      atomicExch(&counters[SCHED_DONE], 0);
    }
  }
}

// Activations [rows, K] bf16, box 64 x ar (a stage's A tile).
bool map_rows(CUtensorMap* m, const void* p, int rows, int K, int ar) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t str[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(ar)};
  return moe_host::encode_bf16_sw128(m, p, 2, dims, str, box);
}

// fp32 outputs [rows, cols], the target of the w2 pass's TMA stores: box of 32
// columns (128 bytes, one swizzle row) x 32 rows.
bool map_out_f32(CUtensorMap* m, const void* p, int rows, int cols) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t str[1] = {static_cast<cuuint64_t>(cols) * 4};
  const cuuint32_t box[2] = {32, 32};
  return moe_host::encode_f32_sw128(m, p, 2, dims, str, box);
}

// fp16 outputs [rows, cols]: box of 64 columns (128 bytes) x 32 rows.
bool map_out_f16(CUtensorMap* m, const void* p, int rows, int cols) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t str[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, 32};
  return moe_host::encode_f16_sw128(m, p, 2, dims, str, box);
}

}  // namespace

namespace moe_host {

size_t experts_ws_bytes() {
  return sizeof(int) * COUNTER_INTS + PARTIAL_BYTES * 4 * static_cast<size_t>(num_sms());
}

namespace {

// Every instance of the kernel has this signature.
using GemmFn = decltype(&grouped_gemm_kernel<EPI_SWIGLU, false, false, BM>);

// The kernels of both passes for one A-tile height (AR rows).
template <int AR>
void pick_kernels(bool shared, bool y_f16, GemmFn* k1, GemmFn* k2) {
  *k1 = shared ? grouped_gemm_kernel<EPI_SWIGLU, true, false, AR>
               : grouped_gemm_kernel<EPI_SWIGLU, false, false, AR>;
  *k2 = y_f16 ? (shared ? grouped_gemm_kernel<EPI_SCALE, true, true, AR>
                        : grouped_gemm_kernel<EPI_SCALE, false, true, AR>)
              : (shared ? grouped_gemm_kernel<EPI_SCALE, true, false, AR>
                        : grouped_gemm_kernel<EPI_SCALE, false, false, AR>);
}

}  // namespace

cudaError_t launch_experts_tc(const void* x_packed, const int32_t* offsets,
                              const float* packed_w, const void* w13, const void* w2, int N,
                              int H, int I, int E, void* h, void* y, bool y_f16,
                              const SharedGroup* sh, void* ws, size_t ws_bytes, int32_t* status,
                              cudaStream_t s, const char** why) {
  // A tile of at most 32 rows needs only 32 rows of A per stage: every
  // expert has at most N rows, the shared expert T2.
  const int T2 = sh ? sh->T : 0, Is = sh ? sh->I : 0;
  const bool short_a = N <= 32 && T2 <= 32;
  const int ar = short_a ? 32 : BM;
  // The shared-expert group is compiled in only where it is used.
  GemmFn k1, k2;
  if (short_a)
    pick_kernels<32>(sh != nullptr, y_f16, &k1, &k2);
  else
    pick_kernels<BM>(sh != nullptr, y_f16, &k1, &k2);
  const size_t smem = short_a ? Ring<32>::SMEM : Ring<BM>::SMEM;
  cudaError_t e1 = ensure_smem(reinterpret_cast<const void*>(k1), static_cast<int>(smem));
  if (e1 != cudaSuccess) return e1;
  e1 = ensure_smem(reinterpret_cast<const void*>(k2), static_cast<int>(smem));
  if (e1 != cudaSuccess) return e1;
  const int nmap = N > 0 ? N : 1;           // a map needs one row; no tile reads it when N == 0
  CUtensorMap mA1, mB1, mA2, mB2, mA1_64, mA1_32, mA2_64, mA2_32;
  bool ok = map_rows(&mA1, x_packed, nmap, H, ar) && map_rows(&mA2, h, nmap, I, ar) &&
            map_rows(&mA1_64, x_packed, nmap, H, 64) && map_rows(&mA1_32, x_packed, nmap, H, 32) &&
            map_rows(&mA2_64, h, nmap, I, 64) && map_rows(&mA2_32, h, nmap, I, 32);
  {
    // w13 as [2E][I][H]: one box = 128 gate rows + the matching 128 up rows.
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(I),
                                static_cast<cuuint64_t>(2) * E};
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(H) * 2,
                               static_cast<cuuint64_t>(I) * H * 2};
    const cuuint32_t box[3] = {BK, BN / 2, 2};
    ok = ok && encode_bf16_sw128(&mB1, w13, 3, dims, str, box);
  }
  {
    // w2 as [E*H][I]
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(I), static_cast<cuuint64_t>(E) * H};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(I) * 2};
    const cuuint32_t box[2] = {BK, BN};
    ok = ok && encode_bf16_sw128(&mB2, w2, 2, dims, str, box);
  }
  // The shared expert's maps (x [T][H], w13s as [2][Is][H], h_s [T][Is], w2s [H][Is]);
  // without one the routed maps stand in, unread.
  CUtensorMap sA1 = mA1, sB1 = mB1, sA2 = mA2, sB2 = mB2;
  if (sh) {
    ok = ok && map_rows(&sA1, sh->x, T2, H, ar) && map_rows(&sA2, sh->h, T2, Is, ar);
    const cuuint64_t d1[3] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(Is), 2};
    const cuuint64_t s1[2] = {static_cast<cuuint64_t>(H) * 2,
                              static_cast<cuuint64_t>(Is) * H * 2};
    const cuuint32_t b1[3] = {BK, BN / 2, 2};
    ok = ok && encode_bf16_sw128(&sB1, sh->w13, 3, d1, s1, b1);
    const cuuint64_t d2[2] = {static_cast<cuuint64_t>(Is), static_cast<cuuint64_t>(H)};
    const cuuint64_t s2[1] = {static_cast<cuuint64_t>(Is) * 2};
    const cuuint32_t b2[2] = {BK, BN};
    ok = ok && encode_bf16_sw128(&sB2, sh->w2, 2, d2, s2, b2);
  }
  // the w2 pass's outputs (the shared expert's own, or the routed map standing in)
  auto map_out = y_f16 ? map_out_f16 : map_out_f32;
  CUtensorMap mY, sY;
  ok = ok && map_out(&mY, y, nmap, H);
  sY = mY;
  if (sh) ok = ok && map_out(&sY, sh->y, T2, H);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)";
    return cudaErrorInvalidValue;
  }
  // Split-K needs the workspace: counters, then 128 KiB partial slots.
  int* counters = nullptr;
  float* partials = nullptr;
  int max_units = 0;
  const size_t cbytes = sizeof(int) * COUNTER_INTS;
  if (ws != nullptr && ws_bytes >= cbytes + PARTIAL_BYTES) {
    counters = static_cast<int*>(ws);
    partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + cbytes);
    max_units = static_cast<int>(std::min<size_t>((ws_bytes - cbytes) / PARTIAL_BYTES, 1 << 20));
  }
  const int sms = num_sms();
  // Feature tiles of pass 1: 128 features each, the last one possibly half full.
  const int ntw1 = (I + BN / 2 - 1) / (BN / 2);
  const int ntw1s = (Is + BN / 2 - 1) / (BN / 2);
  int g1 = sms, g2 = sms;
  if (counters == nullptr) {   // no split possible: never more CTAs than tiles
    const int mt_bound = (N + BM - 1) / BM + E;
    const int mt2 = (T2 + BM - 1) / BM;
    g1 = std::max(1, std::min(sms, mt_bound * ntw1 + mt2 * ntw1s));
    g2 = std::max(1, std::min(sms, (mt_bound + mt2) * (H / BN)));
  }
  const float* no_w = nullptr;
  const uint64_t wait_ns = main_wait_budget_ns();
  cudaError_t err = launch_pdl(k1, dim3(g1), dim3(NTHREADS), smem, s, 0, mA1, mA1_64, mA1_32,
                               mB1, sA1, sB1,
                               mY, sY, offsets, E, H, ntw1, 2 * I, no_w, h, I, T2, H, ntw1s,
                               sh ? sh->h : nullptr, Is, counters, partials, max_units, status,
                               wait_ns);
  if (err != cudaSuccess) return err;
  return launch_pdl(k2, dim3(g2), dim3(NTHREADS), smem, s, 0, mA2, mA2_64, mA2_32, mB2, sA2,
                    sB2, mY, sY,
                    offsets, E, I, H / BN, H, packed_w, y, H, T2, Is, H / BN,
                    sh ? sh->y : nullptr, H, counters, partials, max_units, status, wait_ns);
}

}  // namespace moe_host
