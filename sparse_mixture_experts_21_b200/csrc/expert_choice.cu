// Expert-choice routing: every expert takes the C tokens with the largest affinity.
//
// The Practice page ("路由的数学形式", last paragraphs) and the landscape page (§0)
// describe expert-choice routing: each expert picks its top-C tokens by its own
// capacity, so experts are exactly full and no token is dropped by capacity (a
// token may be picked by no expert or by several).  Readings: affinity = the
// token-choice router's (moe_route_scores writes it expert-major), equal scores
// go to the lower token index, the gate weight of a picked pair is its affinity,
// an expert's rows are its picked tokens in ascending token order.
//
//   ec_select   one CTA per expert: MSB-first radix select over the float bits of
//               its affinity column (non-negative floats order like their bit
//               patterns) finds the C-th largest value exactly in 4 passes of 8
//               bits; a final pass marks the picks (values above the threshold,
//               plus the lowest-index ties) and block scans give their rows in
//               token order.
//   ec_gather   x_perm[row] = x[token_of_row[row]] (one warp per row, 16 B vectors).
//   ec_combine  one warp per token: the experts that picked it, in ascending
//               expert order, y[t] = shared[t] + sum s[t, e] * y_perm[row]; fp32, no
//               atomics on floating point.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace ec {

constexpr int kSelThreads = 1024;

// Exclusive block scan of a 0/1 flag (1024 threads); *total receives the block sum.
__device__ __forceinline__ int block_exscan01(bool flag, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = warp_tot[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    warp_tot[lane] = incl - v;
    if (lane == 31) warp_tot[32] = incl;
  }
  __syncthreads();
  const int r = warp_tot[warp] + in_warp;
  *total = warp_tot[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads)
ec_select_kernel(const float* __restrict__ scores, int64_t T, int C, int N, int32_t* __restrict__ row_of,
                 int32_t* __restrict__ token_of_row, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ n_unpicked) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_mask, s_rem;
  __shared__ int warp_tot[33];
  const int e = blockIdx.x, tid = threadIdx.x;
  const uint32_t* col = reinterpret_cast<const uint32_t*>(scores + (int64_t)e * T);
  if (tid == 0) {
    s_prefix = 0u; s_mask = 0u; s_rem = (uint32_t)C;
    offsets[e] = e * C;
    if (e == 0) { offsets[N] = N * C; if (n_unpicked) *n_unpicked = 0; }
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int64_t t = tid; t < T; t += kSelThreads) {
      const uint32_t key = col[t];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      const uint32_t rem = s_rem;
      uint32_t cum = 0;
      int b = 255;
      for (; b > 0; --b) {
        if (cum + hist[b] >= rem) break;
        cum += hist[b];
      }
      s_rem = rem - cum;
      s_prefix = prefix | ((uint32_t)b << shift);
      s_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t thr = s_prefix;
  const int need_eq = (int)s_rem;           // picks among the values equal to the threshold
  int carry_sel = 0, carry_eq = 0;
  for (int64_t base = 0; base < T; base += kSelThreads) {
    const int64_t t = base + tid;
    const bool valid = t < T;
    const uint32_t key = valid ? col[t] : 0u;
    const bool is_eq = valid && key == thr;
    int tot_eq, tot_sel;
    const int eq_rank = block_exscan01(is_eq, warp_tot, &tot_eq) + carry_eq;
    const bool sel = valid && (key > thr || (is_eq && eq_rank < need_eq));
    const int pos = block_exscan01(sel, warp_tot, &tot_sel) + carry_sel;
    if (valid) {
      const int32_t row = sel ? e * C + pos : -1;
      row_of[(int64_t)e * T + t] = row;
      if (sel) token_of_row[row] = (int32_t)t;
    }
    carry_eq += tot_eq;
    carry_sel += tot_sel;
  }
}

__global__ void __launch_bounds__(256)
ec_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ token_of_row, int64_t R,
                 int nvec, uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp0; r < R; r += nwarps) {
    const uint4* src = x + (int64_t)token_of_row[r] * nvec;
    uint4* dst = x_perm + r * nvec;
    constexpr int U = 4;
    for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nvec) v[u] = ldg_nc16(src + c);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nvec) dst[c] = v[u];
      }
    }
  }
}

constexpr int kCombWarps = 8;
constexpr int kMaxN = 512;

template <typename XT>
__global__ void __launch_bounds__(kCombWarps * 32)
ec_combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ row_of,
                  const float* __restrict__ scores, const uint4* __restrict__ shared_out,
                  uint4* __restrict__ y, int64_t T, int N, int nvec, int32_t* __restrict__ n_unpicked) {
  constexpr int VN = Vec<XT>::N;
  __shared__ int32_t lrow[kCombWarps][kMaxN];
  __shared__ float lw[kCombWarps][kMaxN];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    // the experts that picked t, in ascending expert order
    int cnt = 0;
    for (int e0 = 0; e0 < N; e0 += 32) {
      const int e = e0 + lane;
      const int32_t r = e < N ? row_of[(int64_t)e * T + t] : -1;
      const unsigned bal = __ballot_sync(0xffffffffu, r >= 0);
      if (r >= 0) {
        const int p = cnt + __popc(bal & ((1u << lane) - 1u));
        lrow[wib][p] = r;
        lw[wib][p] = scores[(int64_t)e * T + t];
      }
      cnt += __popc(bal);
    }
    __syncwarp();
    if (cnt == 0 && lane == 0 && n_unpicked) atomicAdd(n_unpicked, 1);
    for (int c = lane; c < nvec; c += 32) {
      float acc[VN];
      if (shared_out) {
        unpack16(ldg_nc16(shared_out + t * nvec + c), acc, XT());
      } else {
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = 0.f;
      }
      for (int j = 0; j < cnt; ++j) {
        float v[VN];
        unpack16(ldg_nc16(y_perm + (int64_t)lrow[wib][j] * nvec + c), v, XT());
        const float wj = lw[wib][j];
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = fmaf(wj, v[i], acc[i]);
      }
      y[t * nvec + c] = pack16(acc, XT());
    }
    __syncwarp();
  }
}

}  // namespace ec

cudaError_t launch_expert_choice(const moe_config_t& c, const void* x, const float* scores, int C,
                                 int32_t* row_of, int32_t* token_of_row, int32_t* offsets, void* x_perm,
                                 int32_t* n_unpicked, cudaStream_t s) {
  const int N = c.n_experts;
  ec::ec_select_kernel<<<N, ec::kSelThreads, 0, s>>>(scores, c.T, C, N, row_of, token_of_row, offsets,
                                                     n_unpicked);
  const int64_t R = (int64_t)N * C;
  if (R > 0) {
    const size_t eb = c.x_dtype == MOE_DTYPE_BF16 ? 2 : 4;
    const int nvec = (int)((size_t)c.d_model * eb / 16);
    const int64_t want = (R + 7) / 8, cap = (int64_t)sm_count() * 8;
    ec::ec_gather_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
        static_cast<const uint4*>(x), token_of_row, R, nvec, static_cast<uint4*>(x_perm));
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_ec(const moe_config_t& c, const void* y_perm, const int32_t* row_of,
                              const float* scores, const void* shared_out, void* y, int32_t* n_unpicked,
                              cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const size_t eb = c.x_dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int nvec = (int)((size_t)c.d_model * eb / 16);
  const int64_t want = (c.T + ec::kCombWarps - 1) / ec::kCombWarps, cap = (int64_t)sm_count() * 8;
  const int grid = (int)(want < cap ? want : cap);
  auto yp = static_cast<const uint4*>(y_perm);
  auto sh = static_cast<const uint4*>(shared_out);
  if (c.x_dtype == MOE_DTYPE_BF16)
    ec::ec_combine_kernel<__nv_bfloat16><<<grid, ec::kCombWarps * 32, 0, s>>>(
        yp, row_of, scores, sh, static_cast<uint4*>(y), c.T, c.n_experts, nvec, n_unpicked);
  else
    ec::ec_combine_kernel<float><<<grid, ec::kCombWarps * 32, 0, s>>>(
        yp, row_of, scores, sh, static_cast<uint4*>(y), c.T, c.n_experts, nvec, n_unpicked);
  return cudaGetLastError();
}

}  // namespace moe
