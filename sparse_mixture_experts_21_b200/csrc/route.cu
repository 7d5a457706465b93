// Fused router: router GEMM -> affinity -> choice-only bias -> group limit ->
// top-k (warp shuffles) -> renormalised weights, plus logsumexp and per-block
// sums of the normalised affinity for the load-balance statistics.
//
// Follows "路由的数学形式：softmax、top-k 与那些必须做的小动作" on the Practice page
// (logits -> softmax -> top-k -> renormalise; bias-free gate), the llm-compass
// "稀疏门控与 Top-k 路由" (g = softmax(TopK(x W_g))) and its "负载均衡：从 aux loss 到
// aux-loss-free" (Top-k over s_i + b_i, weights from s_i).  Group-limited
// pre-selection (the History page's part 四, node-limited routing, no formula
// given): contiguous groups scored by the sum of their top-n selection scores.
//
// Two GEMM front ends share one selection phase (one warp per token, lane l
// holding experts l, l+32, ...):
//  * tensor cores (bf16 x, N <= 256): the fp32 router weight is split exactly
//    into three bf16 pieces W = W_hi + W_mid + W_lo (each piece keeps the next 8
//    mantissa bits), so x W^T = sum over pieces of x W_p^T.  x is bf16, so every
//    product is exact in fp32 and the MMA accumulates in fp32: fp32-equivalent
//    logits from one tcgen05 GEMM with K = 3 d (bf16x3, Henry, Tang & Heinecke,
//    "Leveraging the bfloat16 AI datatype for higher-precision computations",
//    2019).  One CTA per 128 tokens; logits go TMEM -> shared memory.
//  * fp32 FMA (fp32 x, or N > 256): register-tiled SIMT GEMM over d-chunks.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace rt {

struct RouteArgs {
  const float* logit_offset;
  const float* bias;
  int64_t T;
  int N, k, score_fn, renorm, n_groups, topk_groups, group_topn;
  int32_t* topk_idx;
  float* topk_w;
  float* lse;
  float* p_partial;
  float* margin;
  int sink;            // 1: logit column N scores the shared expert (shared-expert sink)
  float* shared_w;     // [T] weight of the shared expert when sink
  float* scores;       // [N, T] affinities, expert-major (expert-choice routing); no top-k
};

// Selection phase: tokens t0 .. t0+TM-1 of the block, logits[tm * ld + e] in
// shared memory.  Writes the per-token outputs and this block's row of p_partial.
//
// One warp per token; lane l holds experts l, l+32, ... (register column i holds
// expert l + 32 i).  Per token: affinity and logsumexp; the group limit (when every
// group is one register column, each lane finds the top groups itself from the
// butterfly-merged column maxima); then each lane sorts its eligible experts by
// selection score once (stable, so the lower expert index stays first on ties), and
// each of the k picks is one warp arg-max over the lanes' list heads, after which
// the winning lane drops its head.  The margin is one more such round.
template <int NV, int WARPS>
__device__ void select_phase(const float* logits, int ld, int TM, int64_t t0, const RouteArgs& a,
                             float* pwarp) {
  // each warp takes two tokens at a time (tm and tm + WARPS) through every step, so
  // the two tokens' dependent chains of warp reductions interleave (one token when a
  // lane holds more than 8 experts: the state of two would not fit in registers)
  constexpr int U = NV <= 8 ? 2 : 1;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int N = a.N, k = a.k;
  float pacc[NV];
  // per-lane constants: validity, group of each column, bias and logit offset
  float bias_r[NV], off_r[NV];
  int gid[NV];
  uint32_t valid_m = 0;
  const int gsz = a.n_groups > 1 ? N / a.n_groups : N;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    pacc[i] = 0.f;
    if (e < N) valid_m |= 1u << i;
    gid[i] = e < N ? e / gsz : 0;
    bias_r[i] = (e < N && a.bias) ? a.bias[e] : 0.f;
    off_r[i] = (e < N && a.logit_offset) ? a.logit_offset[e] : 0.f;
  }
  const bool col_groups = a.n_groups > 1 && gsz == 32 && a.group_topn <= 2;

  for (int tm0 = warp; tm0 < TM; tm0 += U * WARPS) {
    int tmu[U];
    int64_t t[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      tmu[u] = tm0 + u * WARPS;
      t[u] = t0 + tmu[u];
      live[u] = tmu[u] < TM && t[u] < a.T;
    }
    if (!live[0]) break;
    float s[U][NV], q[U][NV];
    float lse[U], s_sh[U], ssum[U];
    {
      float z[U][NV], m[U], z_sh[U], se[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int i = 0; i < NV; ++i)
          z[u][i] = !live[u] ? 0.f
                  : ((valid_m >> i) & 1u) ? logits[tmu[u] * ld + lane + 32 * i] + off_r[i] : -INFINITY;
        // affinity and logsumexp (with the sink, over the N routed logits and the shared one)
        z_sh[u] = (a.sink && live[u]) ? logits[tmu[u] * ld + N] : -INFINITY;
        m[u] = z_sh[u];
#pragma unroll
        for (int i = 0; i < NV; ++i) m[u] = fmaxf(m[u], z[u][i]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) m[u] = warp_max_redux(m[u]);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        se[u] = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          s[u][i] = ((valid_m >> i) & 1u) ? expf(z[u][i] - m[u]) : 0.f;    // exp terms for now
          se[u] += s[u][i];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) se[u] = warp_sum(se[u]);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float ex_sh = a.sink ? expf(z_sh[u] - m[u]) : 0.f;
        se[u] += ex_sh;
        lse[u] = m[u] + logf(se[u]);
        s_sh[u] = 0.f;
        if (a.sink) s_sh[u] = a.score_fn == MOE_SCORE_SOFTMAX ? ex_sh / se[u] : 1.f / (1.f + expf(-z_sh[u]));
        ssum[u] = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const bool v = (valid_m >> i) & 1u;
          if (a.score_fn == MOE_SCORE_SOFTMAX) s[u][i] = v ? s[u][i] / se[u] : 0.f;
          else s[u][i] = v ? 1.f / (1.f + expf(-z[u][i])) : 0.f;
          ssum[u] += s[u][i];
          q[u][i] = v ? s[u][i] + bias_r[i] : -INFINITY;
        }
      }
    }
    // load-balance statistics: routed affinities normalised over the routed experts
    // (softmax probs as they are, or s / sum s)
    if (a.score_fn == MOE_SCORE_SIGMOID || a.sink) {
#pragma unroll
      for (int u = 0; u < U; ++u) ssum[u] = warp_sum(ssum[u]);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (live[u]) {
#pragma unroll
          for (int i = 0; i < NV; ++i) pacc[i] += s[u][i] / ssum[u];
        }
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (live[u]) {
#pragma unroll
          for (int i = 0; i < NV; ++i) pacc[i] += s[u][i];
        }
    }

    if (a.scores) {      // expert-choice routing: the affinity matrix, expert-major
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (live[u]) {
#pragma unroll
          for (int i = 0; i < NV; ++i)
            if ((valid_m >> i) & 1u) a.scores[(int64_t)(lane + 32 * i) * a.T + t[u]] = s[u][i];
          if (lane == 0) a.lse[t[u]] = lse[u];
        }
      continue;
    }

    // group-limited pre-selection: keep bit g = group g kept; gmargin = score of the
    // last kept group minus the best dropped one (ties: lower group index first)
    uint32_t group_keep[U];
    float gmargin[U];
#pragma unroll
    for (int u = 0; u < U; ++u) { group_keep[u] = 0xffffffffu; gmargin[u] = INFINITY; }
    if (a.n_groups > 1) {
      if (col_groups) {
        // each group is one register column: its largest and second largest selection
        // scores (a repeated maximum counts twice) by warp reductions, so every lane
        // knows every group's score and selects the groups itself
        // lane g ends up holding group g's score
        float gl[U];
#pragma unroll
        for (int u = 0; u < U; ++u) gl[u] = -INFINITY;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const uint32_t key = f32_key(q[u][i]);
            const uint32_t k1 = __reduce_max_sync(0xffffffffu, key);
            const uint32_t at_max = __ballot_sync(0xffffffffu, key == k1);
            const uint32_t k2 = __popc(at_max) >= 2 ? k1 : __reduce_max_sync(0xffffffffu, key == k1 ? 0u : key);
            if (lane == i) gl[u] = a.group_topn == 1 ? key_f32(k1) : key_f32(k1) + key_f32(k2);
          }
        }
        // the top groups: one warp arg-max per pick over the lanes' group scores (ties
        // to the lower group index), one more for the margin
#pragma unroll
        for (int u = 0; u < U; ++u) {
          uint32_t kept_mask = 0;
          float last = 0.f;
          for (int r = 0; r <= a.topk_groups && r < a.n_groups; ++r) {
            float v = (lane < a.n_groups && !((kept_mask >> lane) & 1u)) ? gl[u] : -INFINITY;
            int gi = lane;
            warp_argmax_redux(v, gi);
            if (r < a.topk_groups) {
              kept_mask |= 1u << gi;
              last = v;
            } else {
              gmargin[u] = last - v;
            }
          }
          group_keep[u] = kept_mask;
        }
      } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          uint32_t kept_mask = 0;
          float my_gscore = -INFINITY;
          for (int g = 0; g < a.n_groups; ++g) {
            uint32_t taken = 0;
            float gs = 0.f;
            for (int r = 0; r < a.group_topn; ++r) {
              float v = -INFINITY;
              int bi = 0x7fffffff;
#pragma unroll
              for (int i = 0; i < NV; ++i) {
                const int e = lane + 32 * i;
                if (((valid_m >> i) & 1u) && gid[i] == g && !((taken >> i) & 1u) &&
                    (q[u][i] > v || (q[u][i] == v && e < bi))) {
                  v = q[u][i]; bi = e;
                }
              }
              warp_argmax_redux(v, bi);
              gs += v;
              if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
            }
            if (lane == g) my_gscore = gs;
          }
          float last = 0.f;
          for (int r = 0; r <= a.topk_groups && r < a.n_groups; ++r) {
            const bool cand = lane < a.n_groups && !((kept_mask >> lane) & 1u);
            float v = cand ? my_gscore : -INFINITY;
            int gi = cand ? lane : 0x7fffffff;
            warp_argmax_redux(v, gi);
            if (r < a.topk_groups) {
              if (gi != 0x7fffffff) kept_mask |= 1u << gi;
              last = v;
            } else {
              gmargin[u] = last - v;
            }
          }
          group_keep[u] = kept_mask;
        }
      }
    }

    // each lane's eligible experts, sorted by selection score (stable: the lower
    // column, hence the lower expert, first among equal scores)
    float cv[U][NV];
    int ci[U][NV];
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const bool el = ((valid_m >> i) & 1u) && ((group_keep[u] >> gid[i]) & 1u);
        cv[u][i] = el ? q[u][i] : -INFINITY;
        ci[u][i] = i;
      }
#pragma unroll
      for (int x = 1; x < NV; ++x) {
#pragma unroll
        for (int y = x; y > 0; --y) {
          const bool sw = cv[u][y] > cv[u][y - 1];
          const float tv = cv[u][y];
          const int ti = ci[u][y];
          cv[u][y] = sw ? cv[u][y - 1] : cv[u][y];
          ci[u][y] = sw ? ci[u][y - 1] : ci[u][y];
          cv[u][y - 1] = sw ? tv : cv[u][y - 1];
          ci[u][y - 1] = sw ? ti : ci[u][y - 1];
        }
      }
    }
    // k picks, descending, ties to the lower expert index; then the margin's runner-up
    int my_idx[U];
    float kth_q[U], nv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) { my_idx[u] = 0; kth_q[u] = 0.f; nv[u] = -INFINITY; }
    for (int j = 0; j <= k; ++j) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float v = cv[u][0];
        int e = v == -INFINITY ? 0x7fffffff : lane + 32 * ci[u][0];
        warp_argmax_redux(v, e);
        if (j == k) {
          nv[u] = v;
        } else {
          if (e != 0x7fffffff && (e & 31) == lane) {     // the winning lane drops its head
#pragma unroll
            for (int i = 0; i + 1 < NV; ++i) { cv[u][i] = cv[u][i + 1]; ci[u][i] = ci[u][i + 1]; }
            cv[u][NV - 1] = -INFINITY;
          }
          if (lane == j) my_idx[u] = e;
          kth_q[u] = v;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float emargin = (nv[u] == -INFINITY) ? INFINITY : kth_q[u] - nv[u];
      // the affinity of each lane's pick (lanes j < k)
      float my_s = 0.f;
      const int src = lane < k ? (my_idx[u] & 31) : 0;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const float v = __shfl_sync(0xffffffffu, s[u][i], src);
        if (lane < k && (my_idx[u] >> 5) == i) my_s = v;
      }
      const float wsum = warp_sum(lane < k ? my_s : 0.f) + s_sh[u];
      if (live[u]) {
        if (lane < k) {
          a.topk_idx[t[u] * k + lane] = my_idx[u];
          a.topk_w[t[u] * k + lane] = a.renorm ? my_s / wsum : my_s;
        }
        if (lane == 0) {
          a.lse[t[u]] = lse[u];
          if (a.margin) a.margin[t[u]] = fminf(emargin, gmargin[u]);
          if (a.sink) a.shared_w[t[u]] = a.renorm ? s_sh[u] / wsum : s_sh[u];
        }
      }
    }
  }

  // per-block sums of the normalised affinity, fixed order over warps
#pragma unroll
  for (int i = 0; i < NV; ++i) pwarp[(warp * NV + i) * 32 + lane] = pacc[i];
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += WARPS * 32) {
    const int i = e / 32, l = e % 32;
    float sum = 0.f;
    for (int w = 0; w < WARPS; ++w) sum += pwarp[(w * NV + i) * 32 + l];
    a.p_partial[(int64_t)blockIdx.x * N + e] = sum;
  }
}

// ============================================================================
// fp32 FMA front end
// ============================================================================
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
  static constexpr int NV = NP >= 32 ? NP / 32 : 1;   // experts per lane in the selection phase
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
route_simt_kernel(const XT* __restrict__ x, const float* __restrict__ w_gate, int d, RouteArgs a) {
  using S = RouteShape<NP, TM, RM, RN, KS>;
  extern __shared__ __align__(16) float smem[];
  float* xs = smem;                  // [KC][XS]  x chunk, transposed
  float* ws = smem + KC * S::XS;     // [KC][WS]  W_g chunk, transposed
  float* part = smem;                // [KS][TM][NP] after the GEMM (aliases xs/ws)
  float* pwarp = smem + (S::GEMM_FLOATS > S::PART_FLOATS ? S::GEMM_FLOATS : S::PART_FLOATS);

  const int tid = threadIdx.x;
  const int N = a.N + a.sink;     // gate rows (the shared expert's row last)
  const int64_t T = a.T;
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
      float av[RM], bv[RN];
      lds_vec<RM>(xs + kk * S::XS + ty * RM, av);
      lds_vec<RN>(ws + kk * S::WS + tx * RN, bv);
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  // reduce the d-splits in fixed order: logits[tm][e] in part[0]
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
  select_phase<S::NV, S::WARPS>(part, NP, TM, t0, a, pwarp);
}

// ============================================================================
// tensor-core (tcgen05) front end, bf16x3 split of the fp32 router weight
// ============================================================================
// One CTA per 128 tokens.  For every 64-wide slice kt of d, the x tile (16 KB) is
// loaded once and multiplied by the three weight pieces (3 x 4 MMAs of K = 16),
// so x crosses L2 -> shared memory once instead of once per piece.  x tiles and
// weight tiles have rings of their own, each fed by its own producer warp, so an
// x tile (a DRAM miss, the only operand not shared by every CTA) is requested
// A_STAGES slices ahead, independently of the weight tiles (which every CTA reads,
// and which therefore stay in L2).
//
// The tensor cores' fp32 accumulation truncates, so one long accumulation over
// K = 3 d would bias the logits towards zero (about 1e-5 relative at d = 4096).
// Each group of TC_ACC_KT slices (24 MMA steps) therefore starts a fresh TMEM
// accumulator, and drain warps add the group's result into fp32 registers with
// round-to-nearest: the truncation spans the 24 MMA steps of one group only.
constexpr int TC_TM = 128;          // tokens per CTA (MMA M)
constexpr int TC_BK = 64;           // K per slice: one 128-byte swizzle row of bf16
constexpr int TC_A_STAGES = 4;      // x tiles in flight
constexpr int TC_B_RING = 128 * 1024;   // bytes of weight-tile ring
constexpr int TC_ACC_KT = 2;        // slices per fresh accumulator
constexpr int TC_THREADS = 384;     // warp 0 x loads, 1 MMA, 2 weight loads, 4..11 drain; all 12 select
constexpr int TC_WARPS = TC_THREADS / 32;

template <int NP>
struct TcRouteShape {
  static constexpr int A_BYTES = TC_TM * TC_BK * 2;
  static constexpr int B_BYTES = NP * TC_BK * 2;
  static constexpr int B_STAGES = TC_B_RING / B_BYTES > 8 ? 8 : TC_B_RING / B_BYTES;
  static constexpr int RING_BYTES = TC_A_STAGES * A_BYTES + B_STAGES * B_BYTES;
  static constexpr int LD = NP + 1;                           // logits row stride (floats)
  static constexpr int LOGIT_BYTES = TC_TM * LD * 4;
  static constexpr int MAIN_BYTES = RING_BYTES > LOGIT_BYTES ? RING_BYTES : LOGIT_BYTES;
  static constexpr int NV = NP >= 32 ? NP / 32 : 1;
  static constexpr int PWARP_BYTES = TC_WARPS * NV * 32 * 4;
  static constexpr int ACC_COLS = NP < 32 ? 32 : NP;          // TMEM columns per accumulator
  static constexpr int NBUF = 512 / ACC_COLS >= 4 ? 4 : 512 / ACC_COLS;
  static constexpr int TMEM_COLS = NBUF * ACC_COLS;
  static constexpr int DRAIN_WARPS = NP >= 32 ? 8 : 4;
  static constexpr int CPW = NP >= 32 ? NP / 2 : NP;          // columns per drain warp
  static constexpr size_t SMEM = 1024 + MAIN_BYTES + PWARP_BYTES + 512;
};

// Wsplit[e, p * dpad + c] = piece p of W_g[e, c] (zero past N rows / d columns).
__global__ void __launch_bounds__(256)
split_gate_kernel(const float* __restrict__ w_gate, int N, int d, int NP, int dpad,
                  __nv_bfloat16* __restrict__ wsplit) {
  const int64_t n = (int64_t)NP * dpad;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / dpad), c = (int)(i % dpad);
    const float w = (e < N && c < d) ? w_gate[(int64_t)e * d + c] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __nv_bfloat16* row = wsplit + (int64_t)e * 3 * dpad;
    row[c] = hi;
    row[dpad + c] = mid;
    row[2 * dpad + c] = lo;
  }
}

// After an abort, wait (bounded) for the copies this producer issued into the last
// min(issued, STAGES) stages, so none is still writing shared memory at exit.
__device__ __forceinline__ void drain_own_copies(uint64_t* full, int STAGES, uint32_t stage, uint32_t phase,
                                                 int issued) {
  for (int i = 1; i <= min(issued, STAGES); ++i) {
    const int st = ((int)stage - i + 2 * STAGES) % STAGES;
    mbar_wait(&full[st], ((int)stage - i < 0) ? (phase ^ 1u) : phase);
  }
}

template <int NP>
__global__ void __launch_bounds__(TC_THREADS, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                int d, int dpad, RouteArgs a) {
  using S = TcRouteShape<NP>;
  constexpr int AS = TC_A_STAGES, BS = S::B_STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* a_ring = smem;                                     // [AS][A_BYTES]
  uint8_t* b_ring = smem + AS * S::A_BYTES;                   // [BS][B_BYTES]
  float* logits = reinterpret_cast<float*>(smem);             // after the main loop
  float* pwarp = reinterpret_cast<float*>(smem + S::MAIN_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::MAIN_BYTES + S::PWARP_BYTES);
  uint64_t* afull = bars;                           // [AS]
  uint64_t* aempty = afull + AS;                    // [AS]
  uint64_t* bfull = aempty + AS;                    // [BS]
  uint64_t* bempty = bfull + BS;                    // [BS]
  uint64_t* tfull = bempty + BS;                    // [NBUF]
  uint64_t* tempty = tfull + S::NBUF;               // [NBUF]
  uint64_t* mma_done = tempty + S::NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * TC_TM;
  const int nkt = dpad / TC_BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < AS; ++s) { mbar_init(&afull[s], 1); mbar_init(&aempty[s], 1); }
    for (int s = 0; s < BS; ++s) { mbar_init(&bfull[s], 1); mbar_init(&bempty[s], 1); }
    for (int b = 0; b < S::NBUF; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], S::DRAIN_WARPS); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto bounded_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const long long c0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
      if (*abort_flag) return false;
      if (clock64() - c0 > kWaitLimitCycles) { flag_timeout(); *abort_flag = 1; return false; }
    }
    return true;
  };

  if (warp == 0) {
    // ---------------- x tiles: one per slice
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      for (int kt = 0; kt < nkt; ++kt) {
        if (!bounded_wait(&aempty[stage], phase ^ 1u)) {
          drain_own_copies(afull, AS, stage, phase, issued);
          break;
        }
        mbar_arrive_expect_tx(&afull[stage], S::A_BYTES);
        tma_load_2d(&tmX, a_ring + (size_t)stage * S::A_BYTES, &afull[stage], kt * TC_BK, (int32_t)t0);
        ++issued;
        if (++stage == AS) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 2) {
    // ---------------- weight tiles: three pieces per slice
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int kt = 0; kt < nkt && ok; ++kt) {
        for (int p = 0; p < 3; ++p) {
          if (!bounded_wait(&bempty[stage], phase ^ 1u)) {
            drain_own_copies(bfull, BS, stage, phase, issued);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bfull[stage], S::B_BYTES);
          tma_load_2d(&tmW, b_ring + (size_t)stage * S::B_BYTES, &bfull[stage], p * dpad + kt * TC_BK, 0);
          ++issued;
          if (++stage == BS) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(TC_TM, NP < 16 ? 16 : NP);
      uint32_t as = 0, aph = 0, bs = 0, bph = 0;
      bool ok = true;
      for (int kt = 0; kt < nkt && ok; ++kt) {
        const int grp = kt / TC_ACC_KT;
        const bool first = kt % TC_ACC_KT == 0;
        const bool last = kt % TC_ACC_KT == TC_ACC_KT - 1 || kt == nkt - 1;
        const int buf = grp % S::NBUF;
        const uint32_t use = (uint32_t)(grp / S::NBUF) & 1u;
        if (first && !bounded_wait(&tempty[buf], use ^ 1u)) break;
        if (!bounded_wait(&afull[as], aph)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(a_ring + (size_t)as * S::A_BYTES);
        const uint32_t d_tmem = tmem_base + buf * S::ACC_COLS;
        for (int p = 0; p < 3; ++p) {
          if (!bounded_wait(&bfull[bs], bph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t b_addr = smem_u32(b_ring + (size_t)bs * S::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)
            umma_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                     (first && p == 0 && kk == 0) ? 0u : 1u);
          umma_commit(&bempty[bs]);
          if (++bs == BS) { bs = 0; bph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&aempty[as]);
        if (++as == AS) { as = 0; aph ^= 1u; }
        if (last) umma_commit(&tfull[buf]);
      }
      // every MMA of this CTA has finished once this barrier flips
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else if (warp >= 4 && warp < 4 + S::DRAIN_WARPS) {
    // ---------------- drain: TMEM lanes 32 (warp % 4) .. +31, columns [c0, c0 + CPW)
    const int q = warp & 3;
    const int c0 = ((warp - 4) / 4) * S::CPW;
    float acc[S::CPW];
#pragma unroll
    for (int i = 0; i < S::CPW; ++i) acc[i] = 0.f;
    bool ok = true;
    const int ngrp = (nkt + TC_ACC_KT - 1) / TC_ACC_KT;
    for (int grp = 0; grp < ngrp && ok; ++grp) {
      const int buf = grp % S::NBUF;
      const uint32_t use = (uint32_t)(grp / S::NBUF) & 1u;
      ok = bounded_wait(&tfull[buf], use);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * S::ACC_COLS + c0;
#pragma unroll
      for (int c = 0; c < S::CPW; c += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[c + i] += __uint_as_float(v[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
    if (ok) {
      const int r = q * 32 + lane;
#pragma unroll
      for (int i = 0; i < S::CPW; ++i) logits[r * S::LD + c0 + i] = acc[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
  if (*abort_flag) return;
  select_phase<S::NV, TC_WARPS>(logits, S::LD, TC_TM, t0, a, pwarp);
}

template <int NP, int TM, int RM, int RN, int KS>
cudaError_t launch_simt(const moe_config_t& c, const void* x, const float* wg, const RouteArgs& a,
                        cudaStream_t s) {
  using S = RouteShape<NP, TM, RM, RN, KS>;
  const size_t smem = S::SMEM_FLOATS * sizeof(float);
  const unsigned grid = (unsigned)((c.T + TM - 1) / TM);
  if (c.x_dtype == MOE_DTYPE_BF16) {
    auto kern = route_simt_kernel<NP, TM, RM, RN, KS, __nv_bfloat16>;
    const cudaError_t e = ensure_smem_attr((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kRouteThreads, smem, s>>>(static_cast<const __nv_bfloat16*>(x), wg, c.d_model, a);
  } else {
    auto kern = route_simt_kernel<NP, TM, RM, RN, KS, float>;
    const cudaError_t e = ensure_smem_attr((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kRouteThreads, smem, s>>>(static_cast<const float*>(x), wg, c.d_model, a);
  }
  return cudaGetLastError();
}

template <int NP>
cudaError_t launch_split(const moe_config_t& c, const float* wg, __nv_bfloat16* wsplit, cudaStream_t s) {
  const int d = c.d_model;
  const int dpad = (d + TC_BK - 1) / TC_BK * TC_BK;
  const int64_t n = (int64_t)NP * dpad;
  const int sgrid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  split_gate_kernel<<<sgrid, 256, 0, s>>>(wg, c.n_experts + (c.shared_sink ? 1 : 0), d, NP, dpad, wsplit);
  return cudaGetLastError();
}

template <int NP>
cudaError_t launch_tc(const moe_config_t& c, const void* x, const float* wg, const RouteArgs& a,
                      void* ws, cudaStream_t s) {
  using S = TcRouteShape<NP>;
  const int d = c.d_model;
  const int dpad = (d + TC_BK - 1) / TC_BK * TC_BK;
  __nv_bfloat16* wsplit = static_cast<__nv_bfloat16*>(ws);
  if (wg) {                        // else ws holds the split written by moe_route_prepare
    const cudaError_t e = launch_split<NP>(c, wg, wsplit, s);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap mx, mw;
  if (!make_map_bf16(&mx, x, (uint64_t)c.T, (uint64_t)d, TC_TM) ||
      !make_map_bf16(&mw, wsplit, (uint64_t)NP, (uint64_t)3 * dpad, NP))
    return cudaErrorInvalidValue;
  auto kern = route_tc_kernel<NP>;
  cudaError_t e = ensure_smem_attr((const void*)kern, (int)S::SMEM);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((c.T + TC_TM - 1) / TC_TM);
  kern<<<grid, TC_THREADS, S::SMEM, s>>>(mx, mw, d, dpad, a);
  return cudaGetLastError();
}

}  // namespace rt

int route_np(int n) {
  int np = 8;
  while (np < n) np *= 2;
  return np;
}

static int gate_rows(const moe_config_t& c) { return c.n_experts + (c.shared_sink ? 1 : 0); }

bool route_uses_tc(const moe_config_t& c) {
  return c.x_dtype == MOE_DTYPE_BF16 && gate_rows(c) <= 256;
}

int route_tokens_per_block(const moe_config_t& c) {
  if (route_uses_tc(c)) return rt::TC_TM;
  switch (route_np(gate_rows(c))) {
    case 8: case 16: case 32: case 512: return 32;
    default: return 64;
  }
}

size_t route_workspace_bytes(const moe_config_t& c) {
  if (!route_uses_tc(c)) return 0;
  const int np = route_np(gate_rows(c)) < 16 ? 16 : route_np(gate_rows(c));
  const size_t dpad = (size_t)(c.d_model + rt::TC_BK - 1) / rt::TC_BK * rt::TC_BK;
  return (size_t)np * 3 * dpad * 2;
}

cudaError_t launch_route_prepare(const moe_config_t& c, const float* wg, void* ws, cudaStream_t s) {
  __nv_bfloat16* wsplit = static_cast<__nv_bfloat16*>(ws);
  switch (route_np(gate_rows(c))) {
    case 8: case 16: return rt::launch_split<16>(c, wg, wsplit, s);
    case 32:  return rt::launch_split<32>(c, wg, wsplit, s);
    case 64:  return rt::launch_split<64>(c, wg, wsplit, s);
    case 128: return rt::launch_split<128>(c, wg, wsplit, s);
    case 256: return rt::launch_split<256>(c, wg, wsplit, s);
    default:  return cudaErrorInvalidValue;
  }
}

cudaError_t launch_route(const moe_config_t& c, const void* x, const float* wg, const float* off,
                         const float* bias, int32_t* idx, float* w, float* lse, float* pp,
                         float* margin, float* shared_w, void* ws, cudaStream_t s, float* scores) {
  if (c.T == 0) return cudaSuccess;
  rt::RouteArgs a;
  a.logit_offset = off;
  a.bias = bias;
  a.T = c.T;
  a.N = c.n_experts;
  a.k = c.top_k;
  a.score_fn = c.score_fn;
  a.renorm = c.renorm;
  a.n_groups = c.n_groups;
  a.topk_groups = c.topk_groups;
  a.group_topn = c.group_score_topn;
  a.topk_idx = idx;
  a.topk_w = w;
  a.lse = lse;
  a.p_partial = pp;
  a.margin = margin;
  a.sink = c.shared_sink ? 1 : 0;
  a.shared_w = shared_w;
  a.scores = scores;
  if (route_uses_tc(c)) {
    switch (route_np(gate_rows(c))) {
      case 8: case 16: return rt::launch_tc<16>(c, x, wg, a, ws, s);
      case 32:  return rt::launch_tc<32>(c, x, wg, a, ws, s);
      case 64:  return rt::launch_tc<64>(c, x, wg, a, ws, s);
      case 128: return rt::launch_tc<128>(c, x, wg, a, ws, s);
      case 256: return rt::launch_tc<256>(c, x, wg, a, ws, s);
      default:  return cudaErrorInvalidValue;
    }
  }
  switch (route_np(gate_rows(c))) {
    case 8:   return rt::launch_simt<8, 32, 2, 8, 16>(c, x, wg, a, s);
    case 16:  return rt::launch_simt<16, 32, 2, 8, 8>(c, x, wg, a, s);
    case 32:  return rt::launch_simt<32, 32, 4, 8, 8>(c, x, wg, a, s);
    case 64:  return rt::launch_simt<64, 64, 4, 8, 2>(c, x, wg, a, s);
    case 128: return rt::launch_simt<128, 64, 8, 8, 2>(c, x, wg, a, s);
    case 256: return rt::launch_simt<256, 64, 8, 8, 1>(c, x, wg, a, s);
    case 512: return rt::launch_simt<512, 32, 4, 16, 1>(c, x, wg, a, s);
    default:  return cudaErrorInvalidValue;
  }
}

}  // namespace moe
