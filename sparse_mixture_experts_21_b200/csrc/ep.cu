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

}  // namespace ep

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
