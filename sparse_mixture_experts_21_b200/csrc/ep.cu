// Expert parallelism: the data-path kernels around the all-to-all exchange.
//
// The Practice page ("专家并行与 all-to-all") shards the experts over ranks
// (rank of expert e = e / (N / W)), exchanges the per-rank counts before the
// all-to-all, dispatches each kept (token, expert) row to the rank holding the
// expert, computes there, and sends the results back for the weighted combine.
// The local permutation already orders rows by expert, hence by destination rank,
// so the dispatch send buffer is the permuted rows themselves.  What the exchange
// needs on top:
//
//   ep_plan       from the expert offsets of every rank [W, N + 1] (all-gathered): the
//                 send and receive split sizes, the local expert offsets over the
//                 received rows, and the regroup map taking a received row (source
//                 rank major, then expert, then row) to its place in local-expert
//                 order (expert major, then source rank, then row) -- so each local
//                 expert's rows are contiguous for the grouped GEMM.
//   rows_move     dst[r] = src[map[r]] (gather) or dst[map[r]] = src[r] (scatter)
//                 for r < n (n read on the device), 16-byte vectors, one warp per row.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace ep {

// One block per (source rank s, local expert j): fills the regroup map for the
// rows that rank s sends for local expert j.  Block (0, 0) also writes the splits
// and the local offsets.
__global__ void __launch_bounds__(256)
ep_plan_kernel(const int32_t* __restrict__ offsets_all, int W, int rank, int N, int El,
               int32_t* __restrict__ send_splits, int32_t* __restrict__ recv_splits,
               int32_t* __restrict__ local_offsets, int32_t* __restrict__ regroup_map, int64_t recv_cap) {
  const int s = blockIdx.x / El, j = blockIdx.x % El;
  const int e = rank * El + j;                       // global expert
  // rows rank s2 keeps for expert e2
  auto kept = [&](int s2, int e2) -> int64_t {
    const int32_t* o = offsets_all + (int64_t)s2 * (N + 1);
    return (int64_t)o[e2 + 1] - o[e2];
  };
  __shared__ int64_t s_recv_base, s_src_off, s_loc_base, s_loc_src;
  if (threadIdx.x == 0) {
    // received rows of sources before s, and of experts before j within source s
    int64_t recv_base = 0;
    for (int s2 = 0; s2 < s; ++s2)
      for (int j2 = 0; j2 < El; ++j2) recv_base += kept(s2, rank * El + j2);
    int64_t src_off = 0;
    for (int j2 = 0; j2 < j; ++j2) src_off += kept(s, rank * El + j2);
    // local rows of experts before j (all sources), and of sources before s for expert j
    int64_t loc_base = 0;
    for (int j2 = 0; j2 < j; ++j2)
      for (int s2 = 0; s2 < W; ++s2) loc_base += kept(s2, rank * El + j2);
    int64_t loc_src = 0;
    for (int s2 = 0; s2 < s; ++s2) loc_src += kept(s2, e);
    s_recv_base = recv_base;
    s_src_off = src_off;
    s_loc_base = loc_base;
    s_loc_src = loc_src;
    if (blockIdx.x == 0) {
      for (int r = 0; r < W; ++r) {
        int64_t send = 0, recv = 0;
        for (int j2 = 0; j2 < El; ++j2) {
          send += kept(rank, r * El + j2);
          recv += kept(r, rank * El + j2);
        }
        send_splits[r] = (int32_t)send;
        recv_splits[r] = (int32_t)recv;
      }
      int64_t acc = 0;
      for (int j2 = 0; j2 < El; ++j2) {
        local_offsets[j2] = (int32_t)acc;
        for (int s2 = 0; s2 < W; ++s2) acc += kept(s2, rank * El + j2);
      }
      local_offsets[El] = (int32_t)acc;
    }
  }
  __syncthreads();
  const int64_t cnt = kept(s, e);
  const int64_t q0 = s_recv_base + s_src_off;          // first received row of (s, j)
  const int64_t l0 = s_loc_base + s_loc_src;           // its local row
  for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x)
    if (q0 + i < recv_cap) regroup_map[q0 + i] = (int32_t)(l0 + i);
}

__global__ void __launch_bounds__(256)
rows_move_kernel(const uint4* __restrict__ src, int nvec, const int32_t* __restrict__ map,
                 const int32_t* __restrict__ n_rows, int64_t rows_cap, int scatter, uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t n = n_rows ? min((int64_t)*n_rows, rows_cap) : rows_cap;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp0; r < n; r += nwarps) {
    const int64_t m = map[r];
    const uint4* s = src + (scatter ? r : m) * nvec;
    uint4* d = dst + (scatter ? m : r) * nvec;
    for (int c = lane; c < nvec; c += 32) d[c] = ldg_nc16(s + c);
  }
}

// ---------------------------------------------------------------------------
// The exchange over peer memory: every rank maps every other rank's receive buffer,
// its kernels store its rows straight into the ranks that own their experts and load
// the results back from there.  The caller puts a stream-ordered barrier (a
// collective) between the phases, so no kernel ever waits for another rank's kernel.
// A destination's receive buffer is in local-expert order (expert major, then source
// rank, then row), so its grouped FFN runs on it as it stands -- no regroup pass.
//
//   ep_peer_plan   row_addr[i] for this rank's rows i (expert major, moe_permute's
//                  order): the address of row i in rank d = e / El's receive buffer,
//                  d's rows of local experts before e's, then of sources before this
//                  rank for e, then i - offsets[e]; 0 for rows outside this round
//   ep_peer_push   *row_addr[row_of_slot[t, j]] = x[t]: the permutation's row gather
//                  and the dispatch in one pass, x read once per token (the
//                  expert-ordered copy of x is never written)
//   ep_peer_pull   y_perm[i] = *row_addr[i]
// ---------------------------------------------------------------------------

// One block per expert e of the N.
__global__ void __launch_bounds__(256)
ep_peer_plan_kernel(const int32_t* __restrict__ offsets_round, const int32_t* __restrict__ offsets_own, int W,
                    int rank, int N, int El, const uint64_t* __restrict__ peer_rows, int64_t row_bytes,
                    int64_t recv_cap, uint64_t* __restrict__ row_addr) {
  const int e = blockIdx.x, d = e / El, j = e % El;
  auto kept = [&](int s2, int e2) -> int64_t {
    const int32_t* o = offsets_round + (int64_t)s2 * (N + 1);
    return (int64_t)o[e2 + 1] - o[e2];
  };
  __shared__ int64_t s_base, s_cnt;
  if (threadIdx.x == 0) {
    int64_t base = 0;
    for (int j2 = 0; j2 < j; ++j2)
      for (int s2 = 0; s2 < W; ++s2) base += kept(s2, d * El + j2);
    for (int s2 = 0; s2 < rank; ++s2) base += kept(s2, e);
    s_base = base;
    s_cnt = kept(rank, e);
  }
  __syncthreads();
  const int64_t r0 = offsets_own[e], cnt = (int64_t)offsets_own[e + 1] - r0;
  const uint64_t p = peer_rows[d];
  for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x) {
    uint64_t a = 0;
    if (s_cnt > 0) {
      const int64_t q = s_base + i;
      // a piece is wholly in one round and fits the receive buffer (the host plan's
      // packing); anything else is the caller's error and moves no row
      if (i < s_cnt && q < recv_cap && p) a = p + (uint64_t)(q * row_bytes);
      else flag_invalid_index();
    }
    row_addr[r0 + i] = a;
  }
}

// One warp per token: x[t] is read once and stored to the rows of its slots in
// this round, *row_addr[row_of_slot[t, j]] = x[t] (row_addr 0 or row -1: no store).
__global__ void __launch_bounds__(256)
ep_peer_push_kernel(const uint4* __restrict__ x, int nvec, int64_t T, int k,
                    const int32_t* __restrict__ row_of_slot, const uint64_t* __restrict__ row_addr,
                    int64_t rows_cap) {
  constexpr int U = 2;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    uint64_t a = 0;
    if (lane < k) {
      const int32_t row = row_of_slot[t * k + lane];
      if (row >= 0 && row < rows_cap) a = row_addr[row];
      else if (row >= rows_cap) flag_invalid_index();
    }
    unsigned live = __ballot_sync(0xffffffffu, a != 0);
    if (!live) continue;
    const uint4* src = x + t * nvec;
    for (int c0 = lane; c0 < nvec; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < nvec) v[u] = ldg_nc16(src + c0 + 32 * u);
      for (unsigned m = live; m; m &= m - 1) {
        uint4* dst = reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, a, __ffs(m) - 1));
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (c0 + 32 * u < nvec) dst[c0 + 32 * u] = v[u];
      }
    }
  }
  // the stores reach the peers before anything the stream runs after this kernel
  // (the barrier collective that releases the destinations)
  __threadfence_system();
}

// One warp per row: y_perm[r] = *row_addr[r] for r < min(*n_rows, rows_cap), row_addr[r] != 0.
__global__ void __launch_bounds__(256)
ep_peer_pull_kernel(int nvec, const int32_t* __restrict__ n_rows, int64_t rows_cap,
                    const uint64_t* __restrict__ row_addr, uint4* __restrict__ y_perm) {
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int64_t n = min((int64_t)*n_rows, rows_cap);
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp0; r < n; r += nwarps) {
    const uint64_t a = row_addr[r];
    if (!a) continue;
    const uint4* src = reinterpret_cast<const uint4*>(a);
    uint4* dst = y_perm + r * nvec;
    for (int c0 = lane; c0 < nvec; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < nvec) v[u] = ldg16(src + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < nvec) dst[c0 + 32 * u] = v[u];
    }
  }
}

}  // namespace ep

cudaError_t launch_ep_peer_plan(const int32_t* offsets_round, const int32_t* offsets_own, int W, int rank, int N,
                                const uint64_t* peer_rows, int64_t row_bytes, int64_t recv_cap, uint64_t* row_addr,
                                cudaStream_t s) {
  ep::ep_peer_plan_kernel<<<N, 256, 0, s>>>(offsets_round, offsets_own, W, rank, N, N / W, peer_rows, row_bytes,
                                            recv_cap, row_addr);
  return cudaGetLastError();
}

cudaError_t launch_ep_peer_push(const void* x, int64_t row_bytes, int64_t T, int k, const int32_t* row_of_slot,
                                const uint64_t* row_addr, int64_t rows_cap, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int64_t want = (T + 7) / 8, cap = (int64_t)sm_count() * 8;
  ep::ep_peer_push_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(x), (int)(row_bytes / 16), T, k, row_of_slot, row_addr, rows_cap);
  return cudaGetLastError();
}

cudaError_t launch_ep_peer_pull(int64_t row_bytes, const int32_t* n_rows, int64_t rows_cap, const uint64_t* row_addr,
                                void* y_perm, cudaStream_t s) {
  if (rows_cap == 0) return cudaSuccess;
  const int64_t want = (rows_cap + 7) / 8, cap = (int64_t)sm_count() * 8;
  ep::ep_peer_pull_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      (int)(row_bytes / 16), n_rows, rows_cap, row_addr, static_cast<uint4*>(y_perm));
  return cudaGetLastError();
}

cudaError_t launch_ep_plan(const int32_t* offsets_all, int W, int rank, int N, int32_t* send_splits,
                           int32_t* recv_splits, int32_t* local_offsets, int32_t* regroup_map, int64_t recv_cap,
                           cudaStream_t s) {
  const int El = N / W;
  ep::ep_plan_kernel<<<W * El, 256, 0, s>>>(offsets_all, W, rank, N, El, send_splits, recv_splits, local_offsets,
                                            regroup_map, recv_cap);
  return cudaGetLastError();
}

cudaError_t launch_rows_move(const void* src, int64_t row_bytes, const int32_t* map, const int32_t* n_rows,
                             int64_t rows_cap, int scatter, void* dst, cudaStream_t s) {
  if (rows_cap == 0) return cudaSuccess;
  const int64_t want = (rows_cap + 7) / 8, cap = (int64_t)sm_count() * 8;
  ep::rows_move_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(src), (int)(row_bytes / 16), map, n_rows, rows_cap, scatter,
      static_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace moe
