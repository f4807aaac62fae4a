// Expert-parallel routing table on the device.
//
// metrale ep_dispatch.rs, "EpRoutingTable" / "build_ep_routing_table": the
// row-major [num_tokens, top_k] assignments are split into a local bucket
// (expert id in [local_expert_start, local_expert_end)) and a remote bucket
// (every other id), each bucket holding (token index, global expert id,
// weight) triples in the order the assignments were given.  Expert ids are
// compared as unsigned 32-bit values, as the page's u32 ids are.
//
// A stable two-way partition (stream compaction) of the n = num_tokens *
// top_k flat entries f = t * top_k + j:
//   count   -- CTA b owns entries [b*CHUNK, (b+1)*CHUNK) and writes how many
//              of them are local to ws[b]  (skipped when one CTA covers all);
//   scatter -- CTA b adds up ws[0..b) for its first local position (its first
//              remote position is b*CHUNK minus that), each thread takes PER
//              consecutive entries, a block-wide exclusive scan of the
//              threads' local counts gives every entry its position, and the
//              entries are written in order.  The last CTA writes the two
//              bucket sizes.
// Positions grow with f inside each bucket, so the result is unique and
// bit-exact with a sequential walk.
#include <algorithm>

#include "common.cuh"

namespace {

constexpr int EP_NT = 256;                 // threads per CTA
constexpr int EP_PER = 8;                  // consecutive entries per thread
constexpr int EP_CHUNK = EP_NT * EP_PER;   // entries per CTA

__device__ __forceinline__ bool is_local(int32_t id, uint32_t lo, uint32_t hi) {
  const uint32_t u = static_cast<uint32_t>(id);
  return u >= lo && u < hi;
}

__global__ void __launch_bounds__(EP_NT) ep_count_kernel(const int32_t* ids, int n,
                                                         uint32_t lo, uint32_t hi,
                                                         int32_t* __restrict__ block_local) {
  __shared__ int s_warp[EP_NT / 32];
  moe::grid_dep_wait();
  const int base = blockIdx.x * EP_CHUNK;
  int c = 0;
  for (int i = threadIdx.x; i < EP_CHUNK; i += EP_NT) {
    const int f = base + i;
    if (f < n && is_local(moe::ld_prod(ids + f), lo, hi)) ++c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < EP_NT / 32; ++w) t += s_warp[w];
    block_local[blockIdx.x] = t;
  }
  moe::grid_dep_launch();
}

__global__ void __launch_bounds__(EP_NT) ep_scatter_kernel(
    const int32_t* ids, const float* w, int n, int top_k, uint32_t lo,
    uint32_t hi, const int32_t* block_local, int32_t* __restrict__ l_tok,
    int32_t* __restrict__ l_eid, float* __restrict__ l_w, int32_t* __restrict__ r_tok,
    int32_t* __restrict__ r_eid, float* __restrict__ r_w, int32_t* __restrict__ bucket_counts) {
  __shared__ int s_warp[EP_NT / 32];
  __shared__ int s_base;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  moe::grid_dep_wait();
  // First local position of this CTA: the local entries of all earlier CTAs.
  int before = 0;
  if (block_local != nullptr)
    for (int b = threadIdx.x; b < static_cast<int>(blockIdx.x); b += EP_NT)
      before += moe::ld_prod(block_local + b);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  if (lane == 0) s_warp[warp] = before;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
#pragma unroll
    for (int i = 0; i < EP_NT / 32; ++i) t += s_warp[i];
    s_base = t;
  }
  __syncthreads();
  const int cta_local0 = s_base;
  // This thread's PER consecutive entries.
  const int f0 = blockIdx.x * EP_CHUNK + threadIdx.x * EP_PER;
  int32_t id[EP_PER];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < EP_PER; ++i) {
    const int f = f0 + i;
    id[i] = f < n ? moe::ld_prod(ids + f) : 0;
    if (f < n && is_local(id[i], lo, hi)) ++mine;
  }
  // Block-wide exclusive scan of the per-thread local counts.
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  __syncthreads();                           // s_warp reused
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int warp_before = 0;
  for (int i = 0; i < warp; ++i) warp_before += s_warp[i];
  const int local_before = cta_local0 + warp_before + incl - mine;   // local entries before f0
  int lp = local_before;
  int rp = f0 - local_before;                                       // remote entries before f0
#pragma unroll
  for (int i = 0; i < EP_PER; ++i) {
    const int f = f0 + i;
    if (f >= n) break;
    const int32_t tok = f / top_k;
    if (is_local(id[i], lo, hi)) {
      l_tok[lp] = tok;
      l_eid[lp] = id[i];
      l_w[lp] = moe::ld_prod(w + f);
      ++lp;
    } else {
      r_tok[rp] = tok;
      r_eid[rp] = id[i];
      r_w[rp] = moe::ld_prod(w + f);
      ++rp;
    }
  }
  if (blockIdx.x == gridDim.x - 1) {
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int i = 0; i < EP_NT / 32; ++i) t += s_warp[i];
      const int total_local = cta_local0 + t;
      bucket_counts[0] = total_local;
      bucket_counts[1] = n - total_local;
    }
  }
  moe::grid_dep_launch();
}

// Owning rank of expert id under the contiguous split of E experts over R
// ranks, rank q owning [floor(E*q/R), floor(E*(q+1)/R)): the largest q with
// floor(E*q/R) <= id, which is floor((R*(id+1) - 1) / E).
__device__ __forceinline__ int owner_of(int id, int E, int R) {
  return static_cast<int>((static_cast<long long>(R) * (id + 1) - 1) / E);
}

__global__ void __launch_bounds__(256) ep_owner_kernel(const int32_t* ids, int n,
                                                       int E, int R, int32_t* __restrict__ owner,
                                                       int32_t* status) {
  moe::grid_dep_wait();
  for (int f = blockIdx.x * 256 + threadIdx.x; f < n; f += gridDim.x * 256) {
    const int id = moe::ld_prod(ids + f);
    if (id < 0 || id >= E) {
      moe::report(status, MOE_ERR_BAD_INDEX);
      owner[f] = -1;                         // left out by the dispatcher, reported there too
    } else {
      owner[f] = owner_of(id, E, R);
    }
  }
  moe::grid_dep_launch();
}

// local[p] = ids[perm[p]] - (first expert of its owner), for the rows
// p < offsets[R] that a dispatch by owner wrote.
__global__ void __launch_bounds__(256) ep_pack_ids_kernel(const int32_t* ids,
                                                          const int32_t* perm,
                                                          const int32_t* offsets,
                                                          int E, int R,
                                                          int32_t* __restrict__ local) {
  moe::grid_dep_wait();
  const int nrows = moe::ld_prod(offsets + R);
  for (int p = blockIdx.x * 256 + threadIdx.x; p < nrows; p += gridDim.x * 256) {
    const int id = moe::ld_prod(ids + moe::ld_prod(perm + p));
    const int q = owner_of(id, E, R);
    local[p] = id - static_cast<int>(static_cast<long long>(E) * q / R);
  }
  moe::grid_dep_launch();
}

}  // namespace

namespace moe_host {

cudaError_t launch_ep_owner(const int32_t* ids, int n, int E, int R, int32_t* owner,
                            int32_t* status, cudaStream_t s) {
  const int grid = std::max(1, std::min((n + 255) / 256, num_sms() * 4));
  return launch_pdl(ep_owner_kernel, dim3(grid), dim3(256), 0, s, 0, ids, n, E, R, owner, status);
}

cudaError_t launch_ep_pack_ids(const int32_t* ids, const int32_t* perm, const int32_t* offsets,
                               int n, int E, int R, int32_t* local, cudaStream_t s) {
  const int grid = std::max(1, std::min((n + 255) / 256, num_sms() * 4));
  return launch_pdl(ep_pack_ids_kernel, dim3(grid), dim3(256), 0, s, 0, ids, perm, offsets, E, R,
                    local);
}

size_t ep_partition_ws_bytes(long long n) {
  const long long blocks = (n + EP_CHUNK - 1) / EP_CHUNK;
  return std::max<size_t>(static_cast<size_t>(blocks) * sizeof(int32_t), 256);
}

cudaError_t launch_ep_partition(const int32_t* ids, const float* w, int n, int top_k,
                                unsigned lo, unsigned hi, int32_t* l_tok, int32_t* l_eid,
                                float* l_w, int32_t* r_tok, int32_t* r_eid, float* r_w,
                                int32_t* bucket_counts, void* ws, cudaStream_t s) {
  const int blocks = std::max(1, (n + EP_CHUNK - 1) / EP_CHUNK);
  int32_t* bl = nullptr;
  if (blocks > 1) {
    bl = static_cast<int32_t*>(ws);
    cudaError_t e = launch_pdl(ep_count_kernel, dim3(blocks), dim3(EP_NT), 0, s, 0, ids, n, lo,
                               hi, bl);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(ep_scatter_kernel, dim3(blocks), dim3(EP_NT), 0, s, 0, ids, w, n, top_k, lo,
                    hi, static_cast<const int32_t*>(bl), l_tok, l_eid, l_w, r_tok, r_eid, r_w,
                    bucket_counts);
}

}  // namespace moe_host
