// Gate-weighted combine, router statistics and the aux-loss-free bias update.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace cs {

// ---------------------------------------------------------------------------
// Combine: y[t] = shared[t] + sum_{j ascending, row >= 0} w[t,j] * y_perm[row(t,j)]
// (llm-compass "稀疏门控与 Top-k 路由": y = sum_i g_i E_i(x); the Practice page's "共享专家":
// the always-on output is added).  One warp per token, fp32 accumulation in a
// fixed order, 16-byte vectors, no atomics.
// ---------------------------------------------------------------------------
// ADDR: the result of row r is at row_addr[r] (a peer's buffer under expert
// parallelism, 0 when the row has none) instead of y_perm + r.
template <typename XT, int K, int U, bool ADDR = false>
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ row_of_slot,
               const float* __restrict__ topk_w, const uint4* __restrict__ shared_out,
               const float* __restrict__ shared_w, uint4* __restrict__ y, int64_t T, int k,
               int nvec, const uint64_t* __restrict__ row_addr = nullptr) {
  constexpr int VN = Vec<XT>::N;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    int32_t mr = lane < k ? row_of_slot[t * k + lane] : -1;
    const float mw = lane < k ? topk_w[t * k + lane] : 0.f;
    uint64_t ma = 0;
    if constexpr (ADDR) {
      ma = mr >= 0 ? row_addr[mr] : 0;
      if (!ma) mr = -1;
    }
    // a dropped (or padding) slot reads a kept row of the same token with weight 0,
    // so every load below is unconditional and can be issued together
    const unsigned kept = __ballot_sync(0xffffffffu, mr >= 0);
    const float sw = shared_w ? shared_w[t] : 1.f;
    const int any_lane = kept ? __ffs(kept) - 1 : 0;
    const int32_t any_row = __shfl_sync(0xffffffffu, mr, any_lane);
    int32_t rows[K];
    const uint4* src[ADDR ? K : 1];
    float ws[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const int32_t r = __shfl_sync(0xffffffffu, mr, j);
      const float wj = __shfl_sync(0xffffffffu, mw, j);
      rows[j] = r >= 0 ? r : any_row;
      ws[j] = r >= 0 ? wj : 0.f;
      if constexpr (ADDR)
        src[j] = reinterpret_cast<const uint4*>(__shfl_sync(0xffffffffu, ma, r >= 0 ? j : any_lane));
    }
    for (int c0 = lane; c0 < nvec; c0 += 32 * U) {
      float acc[U][VN];
      uint4 v[U][K];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c < nvec && kept) {
#pragma unroll
          for (int j = 0; j < K; ++j) {
            if constexpr (ADDR) v[u][j] = ldg16(src[j] + c);
            else v[u][j] = ldg_nc16(y_perm + (int64_t)rows[j] * nvec + c);
          }
        }
        if (c < nvec && shared_out) {
          unpack16(ldg_nc16(shared_out + t * nvec + c), acc[u], XT());
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[u][i] *= sw;
        } else {
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[u][i] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c >= nvec) continue;
        if (kept) {
#pragma unroll
          for (int j = 0; j < K; ++j) {
            float f[VN];
            unpack16(v[u][j], f, XT());
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[u][i] = fmaf(ws[j], f[i], acc[u][i]);
          }
        }
        y[t * nvec + c] = pack16(acc[u], XT());
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Fixed-order block reduction in double (deterministic).
// ---------------------------------------------------------------------------
template <int NT>
__device__ double block_sum(double v, double* buf) {
  buf[threadIdx.x] = v;
  __syncthreads();
#pragma unroll
  for (int s = NT / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) buf[threadIdx.x] += buf[threadIdx.x + s];
    __syncthreads();
  }
  const double r = buf[0];
  __syncthreads();
  return r;
}

constexpr int kStatThreads = 512;

// Sufficient statistics of one batch, fp64 [3N + 5]: c_e, kept_e, sum_t s-hat_te
// for every expert, then sum_t lse_t^2, T, dropped slots, dropped tokens, near-ties.
// Summing these vectors over data-parallel ranks gives the statistics of the
// concatenated batch.
enum { ST_SUM_Z = 0, ST_T = 1, ST_DROP_SLOTS = 2, ST_DROP_TOKENS = 3, ST_NEAR = 4, ST_TAIL = 5 };

struct StatsArgs {
  const int32_t* counts;
  const int32_t* offsets;
  const float* p_partial;
  int nblk;
  const float* lse;
  const int32_t* n_dropped;
  const float* margin;        // NULL: near-ties not counted (reported as -1)
  float near_tie;
  const double* part_in;      // mode 2
  double* part_out;           // mode 1
  const float* bias;
  int64_t T;
  int k, N;
  float alpha, z_coef;
  moe_stats_t* st;
  float* f_out;
  float* p_out;
  int32_t* counts_out;        // mode 2: the summed counts as int32 (bias update input)
};

// Router statistics (llm-compass "负载均衡": L_aux = alpha N sum f_i P_i; the
// Practice page's load-balance section: 1 before scaling under uniform routing;
// monitoring metrics from the landscape page's 实践要点).  z-loss reading:
// mean_t (logsumexp_e z)^2.  MODE 0: this batch's inputs -> moe_stats_t;
// MODE 1: this batch's inputs -> the sufficient-statistics vector; MODE 2: a
// (summed) vector -> moe_stats_t.  One CTA, fixed-order fp64 reductions.
template <int MODE>
__global__ void __launch_bounds__(kStatThreads) stats_kernel(StatsArgs a) {
  __shared__ double buf[kStatThreads];
  const int e = threadIdx.x, N = a.N;
  double c = 0, kept = 0, psum = 0;
  double zs = 0, near = 0;
  if (MODE != 2) {
    if (e < N) {
      c = a.counts[e];
      kept = a.offsets[e + 1] - a.offsets[e];
      for (int b = 0; b < a.nblk; ++b) psum += a.p_partial[(int64_t)b * N + e];
    }
    for (int64_t t = threadIdx.x; t < a.T; t += kStatThreads) {
      zs += (double)a.lse[t] * a.lse[t];
      if (a.margin) near += a.margin[t] < a.near_tie ? 1.0 : 0.0;
    }
  } else if (e < N) {
    c = a.part_in[e];
    kept = a.part_in[N + e];
    psum = a.part_in[2 * N + e];
  }
  const double sum_z = MODE == 2 ? 0.0 : block_sum<kStatThreads>(zs, buf);
  const double n_near = MODE == 2 ? 0.0 : block_sum<kStatThreads>(near, buf);
  if (MODE == 1) {
    if (e < N) {
      a.part_out[e] = c;
      a.part_out[N + e] = kept;
      a.part_out[2 * N + e] = psum;
    }
    if (threadIdx.x == 0) {
      double* tail = a.part_out + 3 * N;
      tail[ST_SUM_Z] = sum_z;
      tail[ST_T] = (double)a.T;
      tail[ST_DROP_SLOTS] = a.n_dropped[0];
      tail[ST_DROP_TOKENS] = a.n_dropped[1];
      tail[ST_NEAR] = a.margin ? n_near : -1.0;
    }
    return;
  }
  const double* tail = MODE == 2 ? a.part_in + 3 * N : nullptr;
  const double T = MODE == 2 ? tail[ST_T] : (double)a.T;
  double fP = 0, b2 = 0, dead = 0;
  if (e < N) {
    const double P = T > 0 ? psum / T : 0.0;
    const double f = T > 0 ? c / ((double)a.k * T) : 0.0;
    fP = f * P;
    dead = c == 0 ? 1.0 : 0.0;
    if (a.bias) b2 = (double)a.bias[e] * a.bias[e];
    if (a.f_out) a.f_out[e] = (float)f;
    if (a.p_out) a.p_out[e] = (float)P;
    if (a.counts_out) a.counts_out[e] = (int32_t)c;
  }
  const double sum_fP = block_sum<kStatThreads>(fP, buf);
  const double sum_c = block_sum<kStatThreads>(c, buf);
  const double sum_k = block_sum<kStatThreads>(kept, buf);
  const double sum_b2 = block_sum<kStatThreads>(b2, buf);
  const double n_dead = block_sum<kStatThreads>(dead, buf);
  const double mean_c = sum_c / N, mean_k = sum_k / N;
  const double dc = e < N ? (c - mean_c) * (c - mean_c) : 0.0;
  const double dk = e < N ? (kept - mean_k) * (kept - mean_k) : 0.0;
  const double var_c = block_sum<kStatThreads>(dc, buf) / N;
  const double var_k = block_sum<kStatThreads>(dk, buf) / N;
  if (threadIdx.x == 0) {
    const double aux_raw = (double)N * sum_fP;
    const double z = T > 0 ? (MODE == 2 ? tail[ST_SUM_Z] : sum_z) / T : 0.0;
    moe_stats_t* st = a.st;
    st->aux_raw = (float)aux_raw;
    st->aux = (float)(a.alpha * aux_raw);
    st->z = (float)z;
    st->z_loss = (float)(a.z_coef * z);
    st->cv = mean_c > 0 ? (float)(sqrt(var_c) / mean_c) : 0.f;
    st->cv_kept = mean_k > 0 ? (float)(sqrt(var_k) / mean_k) : 0.f;
    st->bias_norm = (float)sqrt(sum_b2);
    st->dead = (int32_t)n_dead;
    st->dropped_slots = MODE == 2 ? (int32_t)tail[ST_DROP_SLOTS] : a.n_dropped[0];
    st->dropped_tokens = MODE == 2 ? (int32_t)tail[ST_DROP_TOKENS] : a.n_dropped[1];
    st->R = (int32_t)sum_k;
    st->near_ties = MODE == 2 ? (int32_t)tail[ST_NEAR] : (a.margin ? (int32_t)n_near : -1);
    st->T = MODE == 2 ? (int64_t)T : a.T;
  }
}

// b[e] += rate * sign(mean(c) - c[e]); the sign is exact: sign(sum c - N c[e]).
// (Practice page BiasBalancedRouter.update_bias; llm-compass "负载均衡".)
__global__ void __launch_bounds__(kStatThreads)
bias_update_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias, int N,
                   float rate, float clamp) {
  __shared__ long long part[kStatThreads];
  part[threadIdx.x] = threadIdx.x < (unsigned)N ? (long long)counts[threadIdx.x] : 0ll;
  __syncthreads();
  for (int s = kStatThreads / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  const long long total = part[0];
  const int e = threadIdx.x;
  if (e < N) {
    const long long diff = total - (long long)N * counts[e];
    const float sgn = diff > 0 ? 1.f : (diff < 0 ? -1.f : 0.f);
    float b = bias[e] + rate * sgn;
    if (clamp > 0.f) b = fminf(fmaxf(b, -clamp), clamp);
    bias[e] = b;
  }
}

// Moving-average controller: ema <- beta ema + (1 - beta) c; b += rate sign(mean(ema) - ema)
// (the landscape page's "bias EMA"; reading of the formula as in the header).
__global__ void __launch_bounds__(kStatThreads)
bias_update_ema_kernel(const int32_t* __restrict__ counts, float* __restrict__ ema, float beta,
                       float* __restrict__ bias, int N, float rate, float clamp) {
  __shared__ double buf[kStatThreads];
  const int e = threadIdx.x;
  double v = 0.0;
  if (e < N) {
    v = (double)beta * (double)ema[e] + (1.0 - (double)beta) * (double)counts[e];
    ema[e] = (float)v;
  }
  const double mean = block_sum<kStatThreads>(e < N ? v : 0.0, buf) / N;
  if (e < N) {
    const double delta = mean - v;
    const float sgn = delta > 0 ? 1.f : (delta < 0 ? -1.f : 0.f);
    float b = bias[e] + rate * sgn;
    if (clamp > 0.f) b = fminf(fmaxf(b, -clamp), clamp);
    bias[e] = b;
  }
}

// Per-sequence share of each expert: part[b, e] = c_be / len_b (one CTA per sequence).
__global__ void __launch_bounds__(256)
seq_load_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ seq_offsets,
                int64_t T, int k, int N, double* __restrict__ part) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  int64_t lo = seq_offsets[blockIdx.x], hi = seq_offsets[blockIdx.x + 1];
  if (lo < 0 || hi > T || lo > hi) {     // a sequence range outside [0, T]: skipped
    if (threadIdx.x == 0) flag_invalid_index();
    lo = hi = 0;
  }
  for (int64_t sl = lo * k + threadIdx.x; sl < hi * k; sl += blockDim.x) {
    const int64_t t = sl / k;
    const int e = checked_expert(topk_idx + t * k, (int)(sl - t * k), N);
    if (e >= 0) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  const double inv = hi > lo ? 1.0 / (double)(hi - lo) : 0.0;
  for (int e = threadIdx.x; e < N; e += blockDim.x)
    part[(int64_t)blockIdx.x * N + e] = hist[e] * inv;
}

// load_e = sum_b part[b, e] in sequence order; b += rate sign(mean(load) - load_e).
__global__ void __launch_bounds__(kStatThreads)
bias_update_seq_kernel(const double* __restrict__ part, int n_seq, float* __restrict__ bias, int N,
                       float rate, float clamp) {
  __shared__ double buf[kStatThreads];
  const int e = threadIdx.x;
  double load = 0.0;
  if (e < N)
    for (int b = 0; b < n_seq; ++b) load += part[(int64_t)b * N + e];
  const double mean = block_sum<kStatThreads>(e < N ? load : 0.0, buf) / N;
  if (e < N) {
    const double delta = mean - load;
    const float sgn = delta > 0 ? 1.f : (delta < 0 ? -1.f : 0.f);
    float b = bias[e] + rate * sgn;
    if (clamp > 0.f) b = fminf(fmaxf(b, -clamp), clamp);
    bias[e] = b;
  }
}

}  // namespace cs


template <typename XT, bool ADDR>
cudaError_t launch_combine_t(const moe_config_t& c, const void* y_perm, const int32_t* row_of_slot,
                             const float* topk_w, const void* shared_out, const float* shared_w,
                             void* y, int grid, int nvec, cudaStream_t s, const uint64_t* row_addr) {
  auto yp = static_cast<const uint4*>(y_perm);
  auto sh = static_cast<const uint4*>(shared_out);
  auto yo = static_cast<uint4*>(y);
#define MOE_COMBINE(KK, UU) \
  cs::combine_kernel<XT, KK, UU, ADDR><<<grid, 256, 0, s>>>(yp, row_of_slot, topk_w, sh, shared_w, yo, c.T, \
                                                            c.top_k, nvec, row_addr)
  switch (c.top_k) {
    case 1: MOE_COMBINE(1, 4); break;
    case 2: MOE_COMBINE(2, 4); break;
    case 3: MOE_COMBINE(3, 2); break;
    case 4: MOE_COMBINE(4, 2); break;
    case 5: MOE_COMBINE(5, 2); break;
    case 6: MOE_COMBINE(6, 2); break;
    case 7: MOE_COMBINE(7, 2); break;
    case 8: MOE_COMBINE(8, 2); break;
    default: MOE_COMBINE(16, 1); break;
  }
#undef MOE_COMBINE
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_config_t& c, const void* y_perm, const int32_t* row_of_slot,
                           const float* topk_w, const void* shared_out, const float* shared_w,
                           void* y, cudaStream_t s, const uint64_t* row_addr) {
  if (c.T == 0) return cudaSuccess;
  const size_t eb = c.x_dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int nvec = (int)((size_t)c.d_model * eb / 16);
  const int64_t want = (c.T + 7) / 8;
  const int64_t cap = (int64_t)sm_count() * 8;
  const int grid = (int)(want < cap ? want : cap);
  if (row_addr) {
    if (c.x_dtype == MOE_DTYPE_BF16)
      return launch_combine_t<__nv_bfloat16, true>(c, nullptr, row_of_slot, topk_w, shared_out, shared_w, y,
                                                   grid, nvec, s, row_addr);
    return launch_combine_t<float, true>(c, nullptr, row_of_slot, topk_w, shared_out, shared_w, y, grid, nvec,
                                         s, row_addr);
  }
  if (c.x_dtype == MOE_DTYPE_BF16)
    return launch_combine_t<__nv_bfloat16, false>(c, y_perm, row_of_slot, topk_w, shared_out, shared_w, y,
                                                  grid, nvec, s, nullptr);
  return launch_combine_t<float, false>(c, y_perm, row_of_slot, topk_w, shared_out, shared_w, y, grid, nvec, s,
                                        nullptr);
}

cudaError_t launch_stats(const moe_config_t& c, int mode, const int32_t* counts, const int32_t* offsets,
                         const float* p_partial, int nblk, const float* lse, const int32_t* n_dropped,
                         const float* margin, float near_tie, const double* part_in, double* part_out,
                         const float* bias, float alpha, float z_coef, moe_stats_t* stats, float* f_out,
                         float* p_out, int32_t* counts_out, cudaStream_t s) {
  cs::StatsArgs a;
  a.counts = counts;
  a.offsets = offsets;
  a.p_partial = p_partial;
  a.nblk = nblk;
  a.lse = lse;
  a.n_dropped = n_dropped;
  a.margin = margin;
  a.near_tie = near_tie;
  a.part_in = part_in;
  a.part_out = part_out;
  a.bias = bias;
  a.T = c.T;
  a.k = c.top_k;
  a.N = c.n_experts;
  a.alpha = alpha;
  a.z_coef = z_coef;
  a.st = stats;
  a.f_out = f_out;
  a.p_out = p_out;
  a.counts_out = counts_out;
  if (mode == 0) cs::stats_kernel<0><<<1, cs::kStatThreads, 0, s>>>(a);
  else if (mode == 1) cs::stats_kernel<1><<<1, cs::kStatThreads, 0, s>>>(a);
  else cs::stats_kernel<2><<<1, cs::kStatThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const moe_config_t& c, const int32_t* counts, float* bias, float rate,
                               float clamp, cudaStream_t s) {
  cs::bias_update_kernel<<<1, cs::kStatThreads, 0, s>>>(counts, bias, c.n_experts, rate, clamp);
  return cudaGetLastError();
}

}  // namespace moe

namespace moe {

cudaError_t launch_bias_update_ema(const moe_config_t& c, const int32_t* counts, float* ema, float beta,
                                   float* bias, float rate, float clamp, cudaStream_t s) {
  cs::bias_update_ema_kernel<<<1, cs::kStatThreads, 0, s>>>(counts, ema, beta, bias, c.n_experts, rate,
                                                            clamp);
  return cudaGetLastError();
}

cudaError_t launch_bias_update_seq(const moe_config_t& c, const int32_t* topk_idx,
                                   const int32_t* seq_offsets, int n_seq, float* bias, float rate,
                                   float clamp, double* ws, cudaStream_t s) {
  if (n_seq > 0)
    cs::seq_load_kernel<<<n_seq, 256, c.n_experts * sizeof(int32_t), s>>>(topk_idx, seq_offsets, c.T,
                                                                         c.top_k, c.n_experts, ws);
  cs::bias_update_seq_kernel<<<1, cs::kStatThreads, 0, s>>>(ws, n_seq, bias, c.n_experts, rate, clamp);
  return cudaGetLastError();
}

}  // namespace moe
