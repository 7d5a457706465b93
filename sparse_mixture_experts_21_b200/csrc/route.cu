// Fused router: fp32 router GEMM -> affinity -> choice-only bias -> group limit
// -> top-k (warp shuffles) -> renormalised weights, plus logsumexp and per-block
// sums of the normalised affinity for the load-balance statistics.
//
// Follows "路由的数学形式：softmax、top-k 与那些必须做的小动作" on the Practice page
// (logits -> softmax -> top-k -> renormalise; bias-free gate), the llm-compass
// "稀疏门控与 Top-k 路由" (g = softmax(TopK(x W_g))) and its "负载均衡：从 aux loss 到
// aux-loss-free" (Top-k over s_i + b_i, weights from s_i).  Group-limited
// pre-selection (the History page's part 四, node-limited routing, no formula
// given): contiguous groups scored by the sum of their top-n selection scores.
//
// One CTA owns TM tokens and all N experts.  Phase 1 is a register-tiled fp32
// SIMT GEMM (x widened from bf16 exactly) with an optional split of each d-chunk
// across thread groups for small N; phase 2 gives each warp one token at a time,
// lane l holding experts l, l+32, ...
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace rt {

constexpr int kRouteThreads = 256;
constexpr int KC = 32;  // d-chunk staged in shared memory per iteration

template <int NP, int TM, int RM, int RN, int KS>
struct RouteShape {
  static constexpr int NTX = NP / RN;            // thread columns (experts)
  static constexpr int NTY = TM / RM;            // thread rows (tokens)
  static_assert(NTX * NTY * KS == kRouteThreads, "thread layout");
  static_assert(KC % KS == 0, "split must divide the chunk");
  static constexpr int XS = TM + 4;              // padded smem strides (floats)
  static constexpr int WS = NP + 4;
  static constexpr int GEMM_FLOATS = KC * XS + KC * WS;
  static constexpr int PART_FLOATS = KS * TM * NP;
  static constexpr int NV = NP >= 32 ? NP / 32 : 1;   // experts per lane in phase 2
  static constexpr int WARPS = kRouteThreads / 32;
  static constexpr int SMEM_FLOATS =
      (GEMM_FLOATS > PART_FLOATS ? GEMM_FLOATS : PART_FLOATS) + WARPS * NV * 32;
};

template <int N>
__device__ __forceinline__ void lds_vec(const float* p, float* out) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      float4 v = *reinterpret_cast<const float4*>(p + i);
      out[i] = v.x; out[i + 1] = v.y; out[i + 2] = v.z; out[i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      float2 v = *reinterpret_cast<const float2*>(p + i);
      out[i] = v.x; out[i + 1] = v.y;
    }
  }
}

template <int NP, int TM, int RM, int RN, int KS, typename XT>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(const XT* __restrict__ x, const float* __restrict__ w_gate,
             const float* __restrict__ logit_offset, const float* __restrict__ bias,
             int64_t T, int d, int N, int k, int score_fn, int renorm, int n_groups,
             int topk_groups, int group_topn, int32_t* __restrict__ topk_idx,
             float* __restrict__ topk_w, float* __restrict__ lse_out,
             float* __restrict__ p_partial, float* __restrict__ margin_out) {
  using S = RouteShape<NP, TM, RM, RN, KS>;
  extern __shared__ __align__(16) float smem[];
  float* xs = smem;                  // [KC][XS]  x chunk, transposed
  float* ws = smem + KC * S::XS;     // [KC][WS]  W_g chunk, transposed
  float* part = smem;                // [KS][TM][NP] after the GEMM (aliases xs/ws)
  float* pwarp = smem + (S::GEMM_FLOATS > S::PART_FLOATS ? S::GEMM_FLOATS : S::PART_FLOATS);

  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int split = tid / (S::NTX * S::NTY);
  const int ty = (tid % (S::NTX * S::NTY)) / S::NTX;
  const int tx = tid % S::NTX;

  float acc[RM][RN];
#pragma unroll
  for (int i = 0; i < RM; ++i)
#pragma unroll
    for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;

  constexpr int XV = Vec<XT>::N;     // x elements per 16-byte vector
  for (int k0 = 0; k0 < d; k0 += KC) {
    // stage x[t0 : t0+TM, k0 : k0+KC] as fp32, transposed
    for (int v = tid; v < TM * (KC / XV); v += kRouteThreads) {
      const int r = v / (KC / XV), c = (v % (KC / XV)) * XV;
      float vals[XV];
      if (t0 + r < T && k0 + c < d) {
        unpack16(ldg_nc16(x + (t0 + r) * (int64_t)d + k0 + c), vals, XT());
      } else {
#pragma unroll
        for (int i = 0; i < XV; ++i) vals[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < XV; ++i) xs[(c + i) * S::XS + r] = vals[i];
    }
    // stage W_g[0 : NP, k0 : k0+KC], transposed
    for (int v = tid; v < NP * (KC / 4); v += kRouteThreads) {
      const int e = v / (KC / 4), c = (v % (KC / 4)) * 4;
      float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < N && k0 + c < d) w4 = *reinterpret_cast<const float4*>(w_gate + (int64_t)e * d + k0 + c);
      ws[(c + 0) * S::WS + e] = w4.x;
      ws[(c + 1) * S::WS + e] = w4.y;
      ws[(c + 2) * S::WS + e] = w4.z;
      ws[(c + 3) * S::WS + e] = w4.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = split; kk < KC; kk += KS) {
      float a[RM], b[RN];
      lds_vec<RM>(xs + kk * S::XS + ty * RM, a);
      lds_vec<RN>(ws + kk * S::WS + tx * RN, b);
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  // ---- reduce the d-splits in fixed order: logits[tm][e] in part[0]
#pragma unroll
  for (int i = 0; i < RM; ++i)
#pragma unroll
    for (int j = 0; j < RN; ++j) part[(split * TM + ty * RM + i) * NP + tx * RN + j] = acc[i][j];
  __syncthreads();
  if constexpr (KS > 1) {
    for (int v = tid; v < TM * NP; v += kRouteThreads) {
      float s = part[v];
#pragma unroll
      for (int q = 1; q < KS; ++q) s += part[q * TM * NP + v];
      part[v] = s;
    }
    __syncthreads();
  }

  // ---- phase 2: one warp per token
  const int warp = tid / 32, lane = tid % 32;
  constexpr int NV = S::NV;
  float pacc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) pacc[i] = 0.f;
  const int gsz = n_groups > 1 ? N / n_groups : N;

  for (int tm = warp; tm < TM; tm += S::WARPS) {
    const int64_t t = t0 + tm;
    if (t >= T) break;
    float z[NV], s[NV], q[NV];
    bool valid[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      valid[i] = e < N;
      z[i] = valid[i] ? part[tm * NP + e] + (logit_offset ? logit_offset[e] : 0.f) : -INFINITY;
    }
    // affinity and logsumexp
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) m = fmaxf(m, z[i]);
    m = warp_max(m);
    float ex[NV], se = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      ex[i] = valid[i] ? expf(z[i] - m) : 0.f;
      se += ex[i];
    }
    se = warp_sum(se);
    const float lse = m + logf(se);
    float ssum = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      if (score_fn == MOE_SCORE_SOFTMAX) s[i] = valid[i] ? ex[i] / se : 0.f;
      else s[i] = valid[i] ? 1.f / (1.f + expf(-z[i])) : 0.f;
      ssum += s[i];
      q[i] = valid[i] ? s[i] + (bias ? bias[lane + 32 * i] : 0.f) : -INFINITY;
    }
    // load-balance statistics: normalised affinity (softmax probs or s / sum s)
    if (score_fn == MOE_SCORE_SIGMOID) {
      ssum = warp_sum(ssum);
#pragma unroll
      for (int i = 0; i < NV; ++i) pacc[i] += s[i] / ssum;
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i) pacc[i] += s[i];
    }

    // group-limited pre-selection
    uint32_t group_keep = 0xffffffffu;
    float gmargin = INFINITY;
    if (n_groups > 1) {
      float my_gscore = -INFINITY;
      for (int g = 0; g < n_groups; ++g) {
        uint32_t taken = 0;
        float gs = 0.f;
        for (int r = 0; r < group_topn; ++r) {
          float v = -INFINITY;
          int bi = 0x7fffffff;
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            const int e = lane + 32 * i;
            if (valid[i] && e / gsz == g && !((taken >> i) & 1u) && (q[i] > v || (q[i] == v && e < bi))) {
              v = q[i]; bi = e;
            }
          }
          warp_argmax(v, bi);
          gs += v;
          if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
        }
        if (lane == g) my_gscore = gs;
      }
      uint32_t kept_mask = 0;
      float last = 0.f;
      for (int r = 0; r <= topk_groups && r < n_groups; ++r) {
        float v = (lane < n_groups && !((kept_mask >> lane) & 1u)) ? my_gscore : -INFINITY;
        int gi = lane < n_groups && !((kept_mask >> lane) & 1u) ? lane : 0x7fffffff;
        warp_argmax(v, gi);
        if (r < topk_groups) {
          if (gi != 0x7fffffff) kept_mask |= 1u << gi;
          last = v;
        } else {
          gmargin = last - v;
        }
      }
      group_keep = kept_mask;
    }

    // top-k over eligible experts, descending, ties to the lower index
    uint32_t taken = 0;
    int my_idx = 0;
    float my_s = 0.f, kth_q = 0.f;
    for (int j = 0; j < k; ++j) {
      float v = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (valid[i] && ((group_keep >> (e / gsz)) & 1u) && !((taken >> i) & 1u) &&
            (q[i] > v || (q[i] == v && e < bi))) {
          v = q[i]; bi = e;
        }
      }
      warp_argmax(v, bi);
      float mine = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if ((bi >> 5) == i) mine = s[i];
      const float sv = __shfl_sync(0xffffffffu, mine, bi & 31);
      if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == j) { my_idx = bi; my_s = sv; }
      kth_q = v;
    }
    // margin to the best eligible expert left out
    float nv = -INFINITY;
    int ni = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (valid[i] && ((group_keep >> (e / gsz)) & 1u) && !((taken >> i) & 1u) &&
          (q[i] > nv || (q[i] == nv && e < ni))) {
        nv = q[i]; ni = e;
      }
    }
    warp_argmax(nv, ni);
    const float emargin = (nv == -INFINITY) ? INFINITY : kth_q - nv;

    const float wsum = warp_sum(lane < k ? my_s : 0.f);
    if (lane < k) {
      topk_idx[t * k + lane] = my_idx;
      topk_w[t * k + lane] = renorm ? my_s / wsum : my_s;
    }
    if (lane == 0) {
      lse_out[t] = lse;
      if (margin_out) margin_out[t] = fminf(emargin, gmargin);
    }
  }

  // ---- per-block sums of the normalised affinity, fixed order over warps
#pragma unroll
  for (int i = 0; i < NV; ++i) pwarp[(warp * NV + i) * 32 + lane] = pacc[i];
  __syncthreads();
  for (int e = tid; e < N; e += kRouteThreads) {
    const int i = e / 32, l = e % 32;
    float sum = 0.f;
    for (int w = 0; w < S::WARPS; ++w) sum += pwarp[(w * NV + i) * 32 + l];
    p_partial[(int64_t)blockIdx.x * N + e] = sum;
  }
}

template <int NP, int TM, int RM, int RN, int KS>
cudaError_t launch_shape(const moe_config_t& c, const void* x, const float* wg, const float* off,
                         const float* bias, int32_t* idx, float* w, float* lse, float* pp,
                         float* margin, cudaStream_t s) {
  using S = RouteShape<NP, TM, RM, RN, KS>;
  const size_t smem = S::SMEM_FLOATS * sizeof(float);
  const unsigned grid = (unsigned)((c.T + TM - 1) / TM);
  if (c.x_dtype == MOE_DTYPE_BF16) {
    auto kern = route_kernel<NP, TM, RM, RN, KS, __nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kRouteThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), wg, off, bias, c.T, c.d_model, c.n_experts, c.top_k,
        c.score_fn, c.renorm, c.n_groups, c.topk_groups, c.group_score_topn, idx, w, lse, pp, margin);
  } else {
    auto kern = route_kernel<NP, TM, RM, RN, KS, float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kRouteThreads, smem, s>>>(
        static_cast<const float*>(x), wg, off, bias, c.T, c.d_model, c.n_experts, c.top_k,
        c.score_fn, c.renorm, c.n_groups, c.topk_groups, c.group_score_topn, idx, w, lse, pp, margin);
  }
  return cudaGetLastError();
}

}  // namespace rt


int route_np(int n) {
  int np = 8;
  while (np < n) np *= 2;
  return np;
}

int route_tokens_per_block(int n) {
  switch (route_np(n)) {
    case 8: case 16: case 32: case 512: return 32;
    default: return 64;
  }
}

cudaError_t launch_route(const moe_config_t& c, const void* x, const float* wg, const float* off,
                         const float* bias, int32_t* idx, float* w, float* lse, float* pp,
                         float* margin, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  switch (route_np(c.n_experts)) {
    case 8:   return rt::launch_shape<8, 32, 2, 8, 16>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 16:  return rt::launch_shape<16, 32, 2, 8, 8>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 32:  return rt::launch_shape<32, 32, 4, 8, 8>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 64:  return rt::launch_shape<64, 64, 4, 8, 2>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 128: return rt::launch_shape<128, 64, 8, 8, 2>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 256: return rt::launch_shape<256, 64, 8, 8, 1>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    case 512: return rt::launch_shape<512, 32, 4, 16, 1>(c, x, wg, off, bias, idx, w, lse, pp, margin, s);
    default:  return cudaErrorInvalidValue;
  }
}

}  // namespace moe
