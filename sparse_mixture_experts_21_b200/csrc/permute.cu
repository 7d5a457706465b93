// Token-order capacity drop and expert-contiguous permutation.
//
// Follows the Practice page's "容量因子、token dropping 与一笔算不清的隐形税" (a hard
// per-expert cap; the earliest occupants are kept so drops are reproducible) and
// "专家并行与 all-to-all：通信才是真正的墙" (slots grouped stably by destination so
// one grouped GEMM covers every expert).  For slot (t, j) choosing expert e:
//   pos(t, j) = #{t' < t : e in idx[t']},  kept iff pos < C,
//   row = offsets[e] + pos,  offsets = exclusive scan of min(c_e, C).
//
// A slot whose expert id is outside [0, N), or repeats an earlier slot of the same
// token, is treated as dropped (row -1, counted in the dropped slots) and never
// indexes anything; the device status word then reads MOE_ERR_INVALID_ARG.
//
// Four launches, all deterministic (integer atomics only, whose result does not
// depend on order):
//   1. hist    per block of kPermuteTokensPerBlock tokens: selections per expert
//   2. scan    per expert: exclusive scan of the block counts in token order,
//              totals c_e, kept counts, offsets (one CTA)
//   3. place   per block: per-expert token bitmaps in shared memory give each
//              slot its rank among earlier tokens of the block -> pos, row
//   4. gather  one warp per token: read x[t] once with 16-byte loads and write
//              it to each of its kept rows
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace pm {

constexpr int TB = kPermuteTokensPerBlock;  // tokens per block
constexpr int kWordsPerExpert = TB / 32;    // token bitmap words per expert

__global__ void __launch_bounds__(256)
permute_hist_kernel(const int32_t* __restrict__ topk_idx, int64_t T, int k, int N,
                    int32_t* __restrict__ blk_counts) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t s0 = (int64_t)blockIdx.x * TB * k;
  const int64_t s1 = min((int64_t)(blockIdx.x + 1) * TB, T) * k;
  for (int64_t sl = s0 + threadIdx.x; sl < s1; sl += blockDim.x) {
    const int64_t t = sl / k;
    const int e = checked_expert(topk_idx + t * k, (int)(sl - t * k), N);
    if (e >= 0) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) blk_counts[(int64_t)blockIdx.x * N + e] = hist[e];
}

// One CTA of 512 threads (N <= 512).  blk_counts becomes the exclusive prefix
// over blocks (the position of each block's first selection of e).
__global__ void __launch_bounds__(512)
permute_scan_kernel(int32_t* __restrict__ blk_counts, int nblk, int N, int64_t T, int k,
                    int64_t capacity, int32_t* __restrict__ counts,
                    int32_t* __restrict__ offsets, int32_t* __restrict__ n_dropped) {
  __shared__ int32_t warp_tot[16];
  const int e = threadIdx.x;
  int32_t kept = 0;
  if (e < N) {
    int32_t run = 0;
    for (int b = 0; b < nblk; ++b) {
      int32_t* p = blk_counts + (int64_t)b * N + e;
      const int32_t c = *p;
      *p = run;
      run += c;
    }
    counts[e] = run;
    kept = (int64_t)run < capacity ? run : (int32_t)capacity;
  }
  // exclusive block scan of kept over experts
  const int lane = e & 31, warp = e >> 5;
  int32_t incl = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t v = lane < 16 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane < 16) warp_tot[lane] = v;  // inclusive totals per warp
  }
  __syncthreads();
  const int32_t base = warp > 0 ? warp_tot[warp - 1] : 0;
  if (e < N) offsets[e] = base + incl - kept;
  if (e == N - 1) {
    const int32_t R = base + incl;
    offsets[N] = R;
    n_dropped[0] = (int32_t)(T * k - R);
    n_dropped[1] = 0;
  }
}

__global__ void __launch_bounds__(256)
permute_place_kernel(const int32_t* __restrict__ topk_idx, int64_t T, int k, int N,
                     int64_t capacity, const int32_t* __restrict__ blk_base,
                     const int32_t* __restrict__ offsets, int32_t* __restrict__ row_of_slot,
                     int32_t* __restrict__ token_of_row, int32_t* __restrict__ n_dropped) {
  extern __shared__ uint32_t bits[];  // [N][kWordsPerExpert]
  __shared__ int32_t blk_dropped;
  for (int i = threadIdx.x; i < N * kWordsPerExpert; i += blockDim.x) bits[i] = 0u;
  if (threadIdx.x == 0) blk_dropped = 0;
  __syncthreads();
  const int64_t tb0 = (int64_t)blockIdx.x * TB;
  const int ntok = (int)min((int64_t)TB, T - tb0);
  for (int i = threadIdx.x; i < ntok * k; i += blockDim.x) {
    const int tl = i / k;
    const int e = checked_expert(topk_idx + (tb0 + tl) * k, i % k, N);
    if (e >= 0) atomicOr(&bits[e * kWordsPerExpert + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  // one thread per token of the block: its k slots
  for (int tl = threadIdx.x; tl < ntok; tl += blockDim.x) {
    const int64_t t = tb0 + tl;
    bool any_kept = false;
    for (int j = 0; j < k; ++j) {
      const int e = checked_expert(topk_idx + t * k, j, N);
      if (e < 0) {                     // invalid or repeated id: a dropped slot
        row_of_slot[t * k + j] = -1;
        continue;
      }
      const uint32_t* be = bits + e * kWordsPerExpert;
      int rank = __popc(be[tl >> 5] & ((1u << (tl & 31)) - 1u));
      for (int w = 0; w < (tl >> 5); ++w) rank += __popc(be[w]);
      const int64_t pos = (int64_t)blk_base[(int64_t)blockIdx.x * N + e] + rank;
      int32_t row = -1;
      if (pos < capacity) {
        row = offsets[e] + (int32_t)pos;
        token_of_row[row] = (int32_t)t;
        any_kept = true;
      }
      row_of_slot[t * k + j] = row;
    }
    if (!any_kept) atomicAdd(&blk_dropped, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0 && blk_dropped) atomicAdd(&n_dropped[1], blk_dropped);
}

// x_perm[row_of_slot[t, j]] = x[t] for every kept slot; x read once per token.
__global__ void __launch_bounds__(256)
permute_gather_kernel(const uint4* __restrict__ x, int64_t T, int k, int nvec,
                      const int32_t* __restrict__ row_of_slot, uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t my_row = lane < k ? row_of_slot[t * k + lane] : -1;
    const uint4* src = x + t * nvec;
    constexpr int U = 4;
    for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nvec) v[u] = ldg_nc16(src + c);
      }
      for (int j = 0; j < k; ++j) {
        const int32_t row = __shfl_sync(0xffffffffu, my_row, j);
        if (row < 0) continue;
        uint4* dst = x_perm + (int64_t)row * nvec;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < nvec) dst[c] = v[u];
        }
      }
    }
  }
}

}  // namespace pm


int permute_blocks(int64_t T) { return (int)((T + pm::TB - 1) / pm::TB); }

size_t permute_workspace_bytes(const moe_config_t& c) {
  return (size_t)permute_blocks(c.T) * (size_t)c.n_experts * sizeof(int32_t);
}

cudaError_t launch_permute(const moe_config_t& c, int64_t capacity, const void* x,
                           const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                           int32_t* row_of_slot, int32_t* token_of_row, void* x_perm,
                           int32_t* n_dropped, int32_t* blk_counts, cudaStream_t s) {
  const int N = c.n_experts, k = c.top_k;
  const int nblk = permute_blocks(c.T);
  if (nblk > 0) {
    pm::permute_hist_kernel<<<nblk, 256, N * sizeof(int32_t), s>>>(topk_idx, c.T, k, N, blk_counts);
  }
  pm::permute_scan_kernel<<<1, 512, 0, s>>>(blk_counts, nblk, N, c.T, k, capacity, counts, offsets,
                                        n_dropped);
  if (nblk == 0) return cudaGetLastError();
  pm::permute_place_kernel<<<nblk, 256, N * pm::kWordsPerExpert * sizeof(uint32_t), s>>>(
      topk_idx, c.T, k, N, capacity, blk_counts, offsets, row_of_slot, token_of_row, n_dropped);
  if (!x_perm || c.T == 0) return cudaGetLastError();
  const size_t eb = c.x_dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int nvec = (int)((size_t)c.d_model * eb / 16);
  const int64_t want_blocks = (c.T + 7) / 8;   // 8 warps (tokens) per block per sweep
  const int grid = (int)(want_blocks < (int64_t)sm_count() * 8 ? want_blocks : (int64_t)sm_count() * 8);
  pm::permute_gather_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), c.T, k, nvec,
                                             row_of_slot, static_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
