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
template <typename XT, int K, int U>
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ row_of_slot,
               const float* __restrict__ topk_w, const uint4* __restrict__ shared_out,
               const float* __restrict__ shared_w, uint4* __restrict__ y, int64_t T, int k,
               int nvec) {
  constexpr int VN = Vec<XT>::N;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t mr = lane < k ? row_of_slot[t * k + lane] : -1;
    const float mw = lane < k ? topk_w[t * k + lane] : 0.f;
    // a dropped (or padding) slot reads a kept row of the same token with weight 0,
    // so every load below is unconditional and can be issued together
    const unsigned kept = __ballot_sync(0xffffffffu, mr >= 0);
    const float sw = shared_w ? shared_w[t] : 1.f;
    const int32_t any_row = kept ? __shfl_sync(0xffffffffu, mr, __ffs(kept) - 1) : 0;
    int32_t rows[K];
    float ws[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const int32_t r = __shfl_sync(0xffffffffu, mr, j);
      const float wj = __shfl_sync(0xffffffffu, mw, j);
      rows[j] = r >= 0 ? r : any_row;
      ws[j] = r >= 0 ? wj : 0.f;
    }
    for (int c0 = lane; c0 < nvec; c0 += 32 * U) {
      float acc[U][VN];
      uint4 v[U][K];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c < nvec && kept) {
#pragma unroll
          for (int j = 0; j < K; ++j) v[u][j] = ldg_nc16(y_perm + (int64_t)rows[j] * nvec + c);
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

// Router statistics (llm-compass "负载均衡": L_aux = alpha N sum f_i P_i; the
// Practice page's load-balance section: 1 before scaling under uniform routing;
// monitoring metrics from the landscape page's 实践要点).  z-loss reading:
// mean_t (logsumexp_e z)^2.
__global__ void __launch_bounds__(kStatThreads)
stats_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
             const float* __restrict__ p_partial, int nblk, const float* __restrict__ lse,
             const int32_t* __restrict__ n_dropped, const float* __restrict__ bias, int64_t T,
             int k, int N, float alpha, float z_coef, moe_stats_t* __restrict__ st,
             float* __restrict__ f_out, float* __restrict__ p_out) {
  __shared__ double buf[kStatThreads];
  const int e = threadIdx.x;
  double c = 0, kept = 0, fP = 0, b2 = 0, dead = 0;
  if (e < N) {
    c = counts[e];
    kept = offsets[e + 1] - offsets[e];
    double P = 0;
    for (int b = 0; b < nblk; ++b) P += p_partial[(int64_t)b * N + e];
    P = T > 0 ? P / (double)T : 0.0;
    const double f = T > 0 ? c / ((double)k * (double)T) : 0.0;
    fP = f * P;
    dead = counts[e] == 0 ? 1.0 : 0.0;
    if (bias) b2 = (double)bias[e] * bias[e];
    if (f_out) f_out[e] = (float)f;
    if (p_out) p_out[e] = (float)P;
  }
  double zs = 0;
  for (int64_t t = threadIdx.x; t < T; t += kStatThreads) zs += (double)lse[t] * lse[t];
  const double sum_fP = block_sum<kStatThreads>(fP, buf);
  const double sum_c = block_sum<kStatThreads>(c, buf);
  const double sum_k = block_sum<kStatThreads>(kept, buf);
  const double sum_b2 = block_sum<kStatThreads>(b2, buf);
  const double n_dead = block_sum<kStatThreads>(dead, buf);
  const double sum_z = block_sum<kStatThreads>(zs, buf);
  const double mean_c = sum_c / N, mean_k = sum_k / N;
  const double dc = e < N ? (c - mean_c) * (c - mean_c) : 0.0;
  const double dk = e < N ? (kept - mean_k) * (kept - mean_k) : 0.0;
  const double var_c = block_sum<kStatThreads>(dc, buf) / N;
  const double var_k = block_sum<kStatThreads>(dk, buf) / N;
  if (threadIdx.x == 0) {
    const double aux_raw = (double)N * sum_fP;
    const double z = T > 0 ? sum_z / (double)T : 0.0;
    st->aux_raw = (float)aux_raw;
    st->aux = (float)(alpha * aux_raw);
    st->z = (float)z;
    st->z_loss = (float)(z_coef * z);
    st->cv = mean_c > 0 ? (float)(sqrt(var_c) / mean_c) : 0.f;
    st->cv_kept = mean_k > 0 ? (float)(sqrt(var_k) / mean_k) : 0.f;
    st->bias_norm = (float)sqrt(sum_b2);
    st->dead = (int32_t)n_dead;
    st->dropped_slots = n_dropped[0];
    st->dropped_tokens = n_dropped[1];
    st->R = offsets[N];
#pragma unroll
    for (int i = 0; i < 5; ++i) st->reserved[i] = 0;
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
                int k, int N, double* __restrict__ part) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t lo = seq_offsets[blockIdx.x], hi = seq_offsets[blockIdx.x + 1];
  for (int64_t sl = lo * k + threadIdx.x; sl < hi * k; sl += blockDim.x) atomicAdd(&hist[topk_idx[sl]], 1);
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


template <typename XT>
cudaError_t launch_combine_t(const moe_config_t& c, const void* y_perm, const int32_t* row_of_slot,
                             const float* topk_w, const void* shared_out, const float* shared_w,
                             void* y, int grid, int nvec, cudaStream_t s) {
  auto yp = static_cast<const uint4*>(y_perm);
  auto sh = static_cast<const uint4*>(shared_out);
  auto yo = static_cast<uint4*>(y);
#define MOE_COMBINE(KK, UU) \
  cs::combine_kernel<XT, KK, UU><<<grid, 256, 0, s>>>(yp, row_of_slot, topk_w, sh, shared_w, yo, c.T, \
                                                      c.top_k, nvec)
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
                           void* y, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const size_t eb = c.x_dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int nvec = (int)((size_t)c.d_model * eb / 16);
  const int64_t want = (c.T + 7) / 8;
  const int64_t cap = (int64_t)sm_count() * 8;
  const int grid = (int)(want < cap ? want : cap);
  if (c.x_dtype == MOE_DTYPE_BF16)
    return launch_combine_t<__nv_bfloat16>(c, y_perm, row_of_slot, topk_w, shared_out, shared_w, y, grid,
                                           nvec, s);
  return launch_combine_t<float>(c, y_perm, row_of_slot, topk_w, shared_out, shared_w, y, grid, nvec, s);
}

cudaError_t launch_stats(const moe_config_t& c, const int32_t* counts, const int32_t* offsets,
                         const float* p_partial, int nblk, const float* lse,
                         const int32_t* n_dropped, const float* bias, float alpha, float z_coef,
                         moe_stats_t* stats, float* f_out, float* p_out, cudaStream_t s) {
  cs::stats_kernel<<<1, cs::kStatThreads, 0, s>>>(counts, offsets, p_partial, nblk, lse, n_dropped, bias,
                                          c.T, c.top_k, c.n_experts, alpha, z_coef, stats, f_out,
                                          p_out);
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
    cs::seq_load_kernel<<<n_seq, 256, c.n_experts * sizeof(int32_t), s>>>(topk_idx, seq_offsets, c.top_k,
                                                                         c.n_experts, ws);
  cs::bias_update_seq_kernel<<<1, cs::kStatThreads, 0, s>>>(ws, n_seq, bias, c.n_experts, rate, clamp);
  return cudaGetLastError();
}

}  // namespace moe
