// C ABI of the MoE layer library: host-side argument checks and launches.
// Every check runs before anything is enqueued, so a rejected call has no effect.
#include <math.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace moe {

// The attribute is a maximum: setting a smaller value lowers it, so each (kernel,
// device) keeps the largest size set so far and only ever raises it.
cudaError_t ensure_smem_attr(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> set_to;   // (kernel, device) -> bytes
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(func, dev);
  const auto it = set_to.find(key);
  if (it != set_to.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) set_to[key] = bytes;
  return e;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 1;
  }
  return cached[dev];
}

namespace capi {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_config(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || (c->d_model % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (c->n_experts < 1 || c->n_experts > 512) return MOE_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > 16) return MOE_ERR_INVALID_ARG;
  if (c->score_fn != MOE_SCORE_SOFTMAX && c->score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c->x_dtype != MOE_DTYPE_F32 && c->x_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->shared_sink != 0 && c->shared_sink != 1) return MOE_ERR_INVALID_ARG;
  if (c->shared_sink && c->n_experts + 1 > 512) return MOE_ERR_INVALID_ARG;
  if (c->capacity_mode < MOE_CAP_DROPLESS || c->capacity_mode > MOE_CAP_CF_K_T_OVER_N_FLOOR)
    return MOE_ERR_INVALID_ARG;
  if (c->capacity_mode != MOE_CAP_DROPLESS && !(c->capacity_factor > 0.0)) return MOE_ERR_INVALID_ARG;
  if (c->n_groups > 1) {
    const int G = c->n_groups;
    if (G > 32 || c->n_experts % G != 0) return MOE_ERR_INVALID_ARG;
    const int gs = c->n_experts / G;
    if (c->topk_groups < 1 || c->topk_groups > G) return MOE_ERR_INVALID_ARG;
    if (c->group_score_topn < 1 || c->group_score_topn > gs) return MOE_ERR_INVALID_ARG;
    if ((int64_t)c->topk_groups * gs < c->top_k) return MOE_ERR_INVALID_ARG;
  }
  if (c->T * (int64_t)c->top_k > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int64_t capacity_of(const moe_config_t& c) {
  switch (c.capacity_mode) {
    case MOE_CAP_CEIL_CF_T_OVER_N:
      return (int64_t)ceil((c.capacity_factor * (double)c.T) / (double)c.n_experts);
    case MOE_CAP_CF_K_T_OVER_N_FLOOR: {
      const double expected = (double)((int64_t)c.top_k * c.T) / (double)c.n_experts;
      const int64_t C = (int64_t)(expected * c.capacity_factor);
      return C > c.top_k ? C : c.top_k;
    }
    default:
      return INT64_MAX;
  }
}

int route_nblk(const moe_config_t& c) {
  const int tm = route_tokens_per_block(c);
  return (int)((c.T + tm - 1) / tm);
}

// The CUDA error behind the last MOE_ERR_CUDA returned to this host thread.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  g_last_cuda_error = e;
  return MOE_ERR_CUDA;
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever arrives on (its own arrival count is 2 and it arrives once), gives up after
// `limit` cycles, records MOE_ERR_DEVICE_TIMEOUT and returns normally.
__global__ void wait_timeout_selftest_kernel(long long limit, int32_t* waited_out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    fence_barrier_init();
    mbar_arrive(&bar);                        // one of two arrivals: the phase never completes
    const bool ok = mbar_wait(&bar, 0, limit);
    if (waited_out) *waited_out = ok ? 1 : 0;
  }
}

}  // namespace capi
}  // namespace moe

using namespace moe;
using namespace moe::capi;

extern "C" {

int moe_capacity(const moe_config_t* cfg, int64_t* capacity) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!capacity) return MOE_ERR_INVALID_ARG;
  *capacity = capacity_of(*cfg);
  return MOE_OK;
}

int moe_route_partials(const moe_config_t* cfg, int32_t* nblk) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!nblk) return MOE_ERR_INVALID_ARG;
  *nblk = route_nblk(*cfg);
  return MOE_OK;
}

int moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const size_t a = permute_workspace_bytes(*cfg), b = route_workspace_bytes(*cfg);
  *bytes = a > b ? a : b;
  return MOE_OK;
}

int moe_route(const moe_config_t* cfg, const void* x, const float* w_gate, const float* logit_offset,
              const float* bias, int32_t* topk_idx, float* topk_w, float* lse, float* p_partial,
              float* margin, float* shared_w, void* ws, size_t ws_bytes, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !topk_idx || !topk_w || !lse || !p_partial) return MOE_ERR_INVALID_ARG;
  if (!w_gate && !route_uses_tc(*cfg)) return MOE_ERR_INVALID_ARG;   // no prepared form on this path
  if (cfg->shared_sink && !shared_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || (w_gate && !aligned16(w_gate))) return MOE_ERR_INVALID_ARG;
  const size_t need = route_workspace_bytes(*cfg);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (!ws || !aligned16(ws))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_route(*cfg, x, w_gate, logit_offset, bias, topk_idx, topk_w, lse, p_partial,
                                margin, cfg->shared_sink ? shared_w : nullptr, ws,
                                static_cast<cudaStream_t>(stream)));
}

int moe_route_prepare_size(const moe_config_t* cfg, size_t* bytes) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = route_workspace_bytes(*cfg);
  return MOE_OK;
}

int moe_route_prepare(const moe_config_t* cfg, const float* w_gate, void* prepared, size_t bytes,
                      void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!route_uses_tc(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!w_gate || !prepared || !aligned16(w_gate) || !aligned16(prepared)) return MOE_ERR_INVALID_ARG;
  if (bytes < route_workspace_bytes(*cfg)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_route_prepare(*cfg, w_gate, prepared, static_cast<cudaStream_t>(stream)));
}

int moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, int32_t* counts,
                int32_t* offsets, int32_t* row_of_slot, int32_t* token_of_row, void* x_perm,
                int32_t* n_dropped, void* ws, size_t ws_bytes, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !n_dropped) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !row_of_slot || !token_of_row || (x_perm && !x)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && x_perm && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  const size_t need = permute_workspace_bytes(*cfg);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (!ws || !aligned16(ws))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_permute(*cfg, capacity_of(*cfg), x, topk_idx, counts, offsets, row_of_slot,
                                  token_of_row, x_perm, n_dropped, static_cast<int32_t*>(ws),
                                  static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap,
                    const int32_t* offsets, int32_t G, const void* w1, const void* w3, const void* w2,
                    int32_t f, void* h_scratch, void* y_rows, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0 || G < 1 || G > 512 || f <= 0 || (f % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (rows_cap > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!x_rows || !w1 || !w3 || !w2 || !h_scratch || !y_rows) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2) ||
      !aligned16(h_scratch) || !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  const int d = cfg->d_model;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->x_dtype == MOE_DTYPE_BF16)
    return from_cuda(launch_ffn_bf16(x_rows, rows_cap, offsets, G, w1, w3, w2, d, f, h_scratch, y_rows, s));
  return from_cuda(launch_ffn_f32(static_cast<const float*>(x_rows), rows_cap, offsets, G,
                                  static_cast<const float*>(w1), static_cast<const float*>(w3),
                                  static_cast<const float*>(w2), d, f, static_cast<float*>(h_scratch),
                                  static_cast<float*>(y_rows), s));
}

int moe_grouped_ffn_shared(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap,
                           const int32_t* offsets, int32_t G, const void* w1, const void* w3, const void* w2,
                           int32_t f, void* h_scratch, void* y_rows, const void* x, int64_t T, const void* ws1,
                           const void* ws3, const void* ws2, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0)
    return moe_grouped_ffn(cfg, x_rows, rows_cap, offsets, G, w1, w3, w2, f, h_scratch, y_rows, stream);
  if (rows_cap < 0 || G < 1 || G > 511 || f <= 0 || (f % 8) != 0 || !offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap + T > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!w1 || !w3 || !w2 || !x || !ws1 || !ws3 || !ws2 || !h_scratch || !y_rows) return MOE_ERR_INVALID_ARG;
  if (rows_cap > 0 && !x_rows) return MOE_ERR_INVALID_ARG;
  if ((x_rows && !aligned16(x_rows)) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2) ||
      !aligned16(h_scratch) || !aligned16(y_rows) || !aligned16(x) || !aligned16(ws1) || !aligned16(ws3) ||
      !aligned16(ws2))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_bf16_shared(x_rows, rows_cap, offsets, G, w1, w3, w2, cfg->d_model, f, h_scratch,
                                          y_rows, x, (int)T, ws1, ws3, ws2, static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_gate_up(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap, const int32_t* offsets,
                            int32_t G, const void* w1, const void* w3, int32_t f, void* h_rows, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < 0 || G < 1 || G > 512 || f <= 0 || (f % 8) != 0 || !offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (rows_cap > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!x_rows || !w1 || !w3 || !h_rows) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w1) || !aligned16(w3) || !aligned16(h_rows)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_bf16_gate_up(x_rows, rows_cap, offsets, G, w1, w3, cfg->d_model, f, h_rows,
                                           static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_down(const moe_config_t* cfg, const void* h_rows, int64_t rows_cap, const int32_t* offsets,
                         int32_t G, const void* w2, int32_t f, void* y_rows, int64_t T, const void* ws2,
                         void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < 0 || T < 0 || G < 1 || G > 511 || f <= 0 || (f % 8) != 0 || !offsets) return MOE_ERR_INVALID_ARG;
  if ((T > 0) != (ws2 != nullptr)) return MOE_ERR_INVALID_ARG;
  if (rows_cap + T == 0) return MOE_OK;
  if (rows_cap + T > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!h_rows || !w2 || !y_rows) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h_rows) || !aligned16(w2) || !aligned16(y_rows) || (ws2 && !aligned16(ws2)))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_bf16_down(h_rows, rows_cap, offsets, G, w2, cfg->d_model, f, y_rows, (int)T, ws2,
                                        static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_gather(const moe_config_t* cfg, const void* x, int64_t T, const int32_t* token_of_row,
                           int64_t rows_cap, const int32_t* offsets, int32_t G, const void* w1, const void* w3,
                           const void* w2, int32_t f, void* h_scratch, void* y_rows, const void* ws1,
                           const void* ws3, const void* ws2, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  // every gathered row chunk lies inside x: whole 64-column steps, ids checked on the device
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 64) != 0) return MOE_ERR_UNSUPPORTED;
  if (T < 0 || rows_cap < 0 || G < 1 || G > 511 || f <= 0 || (f % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (!offsets || !token_of_row) return MOE_ERR_INVALID_ARG;
  const bool shared = ws1 || ws3 || ws2;
  if (shared && (!ws1 || !ws3 || !ws2)) return MOE_ERR_INVALID_ARG;
  if (T == 0 || (rows_cap == 0 && !shared)) return MOE_OK;
  if (rows_cap + (shared ? T : 0) > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!x || !w1 || !w3 || !w2 || !h_scratch || !y_rows) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2) || !aligned16(h_scratch) ||
      !aligned16(y_rows) || (reinterpret_cast<uintptr_t>(token_of_row) & 3u))
    return MOE_ERR_INVALID_ARG;
  if (shared && (!aligned16(ws1) || !aligned16(ws3) || !aligned16(ws2))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_bf16_gather(x, (int)T, token_of_row, rows_cap, offsets, G, w1, w3, w2,
                                          cfg->d_model, f, h_scratch, y_rows, ws1, ws3, ws2,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_quantize_fp8(const void* x, int64_t rows, int32_t cols, int32_t block_rows, uint8_t* q,
                     float* scales, void* stream) {
  if (rows < 0 || cols <= 0 || (cols % 128) != 0 || (block_rows != 1 && block_rows != 128))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return MOE_ERR_INVALID_ARG;
  if (block_rows == 128 && (rows + 127) / 128 * (cols / 128) > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  return from_cuda(launch_quantize_fp8(x, rows, cols, block_rows, q, scales, static_cast<cudaStream_t>(stream)));
}

int moe_permute_fp8(const moe_config_t* cfg, const void* x, const int32_t* row_of_slot, uint8_t* xq_perm,
                    float* xs_perm, uint8_t* xq, float* xs, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 128) != 0) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (row_of_slot && (!xq_perm || !xs_perm)) return MOE_ERR_INVALID_ARG;
  if (!row_of_slot && !xq) return MOE_ERR_INVALID_ARG;
  if ((xq && !xs) || (xq_perm && !aligned16(xq_perm)) || (xq && !aligned16(xq)))
    return MOE_ERR_INVALID_ARG;
  if ((xs_perm && (reinterpret_cast<uintptr_t>(xs_perm) & 3u)) || (xs && (reinterpret_cast<uintptr_t>(xs) & 3u)))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_quant_scatter(x, cfg->T, row_of_slot ? cfg->top_k : 0, cfg->d_model, row_of_slot,
                                        xq_perm, xs_perm, xq, xs, static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_fp8(const moe_config_t* cfg, const uint8_t* xq_rows, const float* xs_rows,
                        int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                        const float* w1s, const uint8_t* w3q, const float* w3s, const uint8_t* w2q,
                        const float* w2s, int32_t f, uint8_t* hq_scratch, float* hs_scratch, void* y_rows,
                        void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0 || G < 1 || G > 512 || f <= 0) return MOE_ERR_INVALID_ARG;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 128) != 0 || (f % 128) != 0)
    return MOE_ERR_UNSUPPORTED;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (rows_cap > (int64_t)INT32_MAX || (int64_t)G * cfg->d_model > (int64_t)INT32_MAX ||
      (int64_t)G * f > (int64_t)INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (!xq_rows || !xs_rows || !w1q || !w1s || !w3q || !w3s || !w2q || !w2s || !hq_scratch || !hs_scratch ||
      !y_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq_rows) || !aligned16(w1q) || !aligned16(w3q) || !aligned16(w2q) || !aligned16(hq_scratch) ||
      !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_fp8(xq_rows, xs_rows, rows_cap, offsets, G, w1q, w1s, w3q, w3s, w2q, w2s,
                                  cfg->d_model, f, hq_scratch, hs_scratch, y_rows,
                                  static_cast<cudaStream_t>(stream)));
}

int moe_quantize_mxfp8(const void* x, int64_t rows, int32_t cols, uint8_t* q, uint8_t* sf, void* stream) {
  if (rows < 0 || cols <= 0 || (cols % 128) != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !sf || !aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7u)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_mx_quant_rows(x, rows, cols, q, sf, static_cast<cudaStream_t>(stream)));
}

int moe_permute_mxfp8(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* row_of_slot,
                      const int32_t* offsets, uint8_t* q_perm, uint8_t* sf_perm, uint8_t* q, uint8_t* sf,
                      void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 128) != 0 || cfg->n_experts > 1024)
    return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (row_of_slot && (!q_perm || !sf_perm || !topk_idx || !offsets)) return MOE_ERR_INVALID_ARG;
  if (!row_of_slot && !q) return MOE_ERR_INVALID_ARG;
  if ((q && !sf) || (q_perm && !aligned16(q_perm)) || (q && !aligned16(q))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_mx_quant_scatter(x, cfg->T, row_of_slot ? cfg->top_k : 0, cfg->d_model,
                                           cfg->n_experts, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q,
                                           sf, static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_mxfp8(const moe_config_t* cfg, const uint8_t* xq_rows, const uint8_t* xsf_rows,
                          int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                          const uint8_t* w1sf, const uint8_t* w3q, const uint8_t* w3sf, const uint8_t* w2q,
                          const uint8_t* w2sf, int32_t f, uint8_t* hq_scratch, uint8_t* hsf_scratch,
                          void* y_rows, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0 || G < 1 || G > 512 || f <= 0) return MOE_ERR_INVALID_ARG;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 128) != 0 || (f % 128) != 0)
    return MOE_ERR_UNSUPPORTED;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (rows_cap > (int64_t)INT32_MAX || (int64_t)G * cfg->d_model > (int64_t)INT32_MAX ||
      (int64_t)G * f > (int64_t)INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (!xq_rows || !xsf_rows || !w1q || !w1sf || !w3q || !w3sf || !w2q || !w2sf || !hq_scratch ||
      !hsf_scratch || !y_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq_rows) || !aligned16(w1q) || !aligned16(w3q) || !aligned16(w2q) || !aligned16(hq_scratch) ||
      !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xsf_rows) || !aligned16(w1sf) || !aligned16(w3sf) || !aligned16(w2sf) || !aligned16(hsf_scratch))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_mx(xq_rows, xsf_rows, rows_cap, offsets, G, w1q, w1sf, w3q, w3sf, w2q, w2sf,
                                 cfg->d_model, f, hq_scratch, hsf_scratch, y_rows,
                                 static_cast<cudaStream_t>(stream)));
}

int moe_quantize_nvfp4(const void* x, int64_t rows, int32_t cols, int32_t tensor_rows, uint8_t* q, uint8_t* sf,
                       float* g, void* stream) {
  if (rows < 0 || cols <= 0 || (cols % 64) != 0 || tensor_rows < 0) return MOE_ERR_INVALID_ARG;
  if (tensor_rows > 0 && (rows % tensor_rows) != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (rows * (int64_t)cols / 8 > ((int64_t)1 << 40)) return MOE_ERR_UNSUPPORTED;
  if (!x || !q || !sf || !aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 3u)) return MOE_ERR_INVALID_ARG;
  if (tensor_rows > 0 && (!g || (reinterpret_cast<uintptr_t>(g) & 3u))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_nv_quant_rows(x, rows, cols, tensor_rows, q, sf, tensor_rows > 0 ? g : nullptr,
                                        static_cast<cudaStream_t>(stream)));
}

int moe_permute_nvfp4(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* row_of_slot,
                      const int32_t* offsets, uint8_t* q_perm, uint8_t* sf_perm, uint8_t* q, uint8_t* sf,
                      void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 256) != 0 || cfg->n_experts > 1024)
    return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (row_of_slot && (!q_perm || !sf_perm || !topk_idx || !offsets)) return MOE_ERR_INVALID_ARG;
  if (!row_of_slot && !q) return MOE_ERR_INVALID_ARG;
  if ((q && !sf) || (q_perm && !aligned16(q_perm)) || (q && !aligned16(q))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_nv_quant_scatter(x, cfg->T, row_of_slot ? cfg->top_k : 0, cfg->d_model,
                                           cfg->n_experts, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q,
                                           sf, static_cast<cudaStream_t>(stream)));
}

int moe_grouped_ffn_nvfp4(const moe_config_t* cfg, const uint8_t* xq_rows, const uint8_t* xsf_rows,
                          int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                          const uint8_t* w1sf, const float* g1, const uint8_t* w3q, const uint8_t* w3sf,
                          const float* g3, const uint8_t* w2q, const uint8_t* w2sf, const float* g2, int32_t f,
                          uint8_t* hq_scratch, uint8_t* hsf_scratch, void* y_rows, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0 || G < 1 || G > 512 || f <= 0) return MOE_ERR_INVALID_ARG;
  if (cfg->x_dtype != MOE_DTYPE_BF16 || (cfg->d_model % 256) != 0 || (f % 256) != 0) return MOE_ERR_UNSUPPORTED;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (rows_cap > (int64_t)INT32_MAX || (int64_t)G * cfg->d_model > (int64_t)INT32_MAX ||
      (int64_t)G * f > (int64_t)INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (!xq_rows || !xsf_rows || !w1q || !w1sf || !g1 || !w3q || !w3sf || !g3 || !w2q || !w2sf || !g2 ||
      !hq_scratch || !hsf_scratch || !y_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq_rows) || !aligned16(w1q) || !aligned16(w3q) || !aligned16(w2q) || !aligned16(hq_scratch) ||
      !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xsf_rows) || !aligned16(w1sf) || !aligned16(w3sf) || !aligned16(w2sf) || !aligned16(hsf_scratch))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(g1) | reinterpret_cast<uintptr_t>(g3) | reinterpret_cast<uintptr_t>(g2)) & 3u)
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ffn_nv(xq_rows, xsf_rows, rows_cap, offsets, G, w1q, w1sf, g1, w3q, w3sf, g3, w2q, w2sf,
                                 g2, cfg->d_model, f, hq_scratch, hsf_scratch, y_rows,
                                 static_cast<cudaStream_t>(stream)));
}

int moe_ep_plan(const int32_t* offsets_all, int32_t world, int32_t rank, int32_t n_experts, int32_t* send_splits,
                int32_t* recv_splits, int32_t* local_offsets, int32_t* regroup_map, int64_t recv_cap, void* stream) {
  if (world < 1 || n_experts < 1 || rank < 0 || rank >= world || (n_experts % world) != 0 || recv_cap < 0)
    return MOE_ERR_INVALID_ARG;
  if (!offsets_all || !send_splits || !recv_splits || !local_offsets || (recv_cap > 0 && !regroup_map))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ep_plan(offsets_all, world, rank, n_experts, send_splits, recv_splits, local_offsets,
                                  regroup_map, recv_cap, static_cast<cudaStream_t>(stream)));
}

int moe_rows_move(const void* src, int64_t row_bytes, const int32_t* map, const int32_t* n_rows, int64_t rows_cap,
                  int32_t scatter, void* dst, void* stream) {
  if (row_bytes <= 0 || (row_bytes % 16) != 0 || rows_cap < 0 || (scatter != 0 && scatter != 1))
    return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (!src || !map || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_rows_move(src, row_bytes, map, n_rows, rows_cap, scatter, dst,
                                    static_cast<cudaStream_t>(stream)));
}

int moe_peer_export(const void* ptr, void* handle) {
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  int64_t off = 0;
  uint8_t* h = static_cast<uint8_t*>(handle);
  const cudaError_t e = peer_export(ptr, h, &off);
  if (e == cudaErrorInvalidValue) return MOE_ERR_INVALID_ARG;
  if (e != cudaSuccess) return from_cuda(e);
  memcpy(h + MOE_PEER_HANDLE_BYTES - 8, &off, 8);
  return MOE_OK;
}

int moe_peer_import(const void* handle, void** ptr) {
  if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
  int64_t off = 0;
  memcpy(&off, static_cast<const uint8_t*>(handle) + MOE_PEER_HANDLE_BYTES - 8, 8);
  if (off < 0) return MOE_ERR_INVALID_ARG;
  *ptr = nullptr;
  return from_cuda(peer_import(static_cast<const uint8_t*>(handle), off, ptr));
}

int moe_peer_close(void* ptr) {
  if (!ptr) return MOE_ERR_INVALID_ARG;
  const int st = peer_close(ptr);
  if (st == 1) return MOE_ERR_INVALID_ARG;
  return from_cuda((cudaError_t)st);
}

int moe_ep_peer_plan(const int32_t* offsets_round, const int32_t* offsets_own, int32_t world, int32_t rank,
                     int32_t n_experts, const uint64_t* peer_rows, int64_t row_bytes, int64_t recv_cap,
                     uint64_t* row_addr, void* stream) {
  if (world < 1 || n_experts < 1 || rank < 0 || rank >= world || (n_experts % world) != 0 || recv_cap < 0 ||
      row_bytes <= 0 || (row_bytes % 16) != 0)
    return MOE_ERR_INVALID_ARG;
  if (!offsets_round || !offsets_own || !peer_rows || !row_addr) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ep_peer_plan(offsets_round, offsets_own, world, rank, n_experts, peer_rows, row_bytes,
                                       recv_cap, row_addr, static_cast<cudaStream_t>(stream)));
}

int moe_ep_peer_dispatch(const moe_config_t* cfg, const void* x, const int32_t* row_of_slot,
                         const uint64_t* row_addr, int64_t rows_cap, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0 || cfg->T == 0) return MOE_OK;
  if (!x || !aligned16(x) || !row_of_slot || !row_addr) return MOE_ERR_INVALID_ARG;
  const int64_t row_bytes = (int64_t)cfg->d_model * (cfg->x_dtype == MOE_DTYPE_BF16 ? 2 : 4);
  return from_cuda(launch_ep_peer_push(x, row_bytes, cfg->T, cfg->top_k, row_of_slot, row_addr, rows_cap,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_ep_peer_collect(const moe_config_t* cfg, const uint64_t* row_addr, const int32_t* n_rows, int64_t rows_cap,
                        void* y_perm, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (rows_cap < 0) return MOE_ERR_INVALID_ARG;
  if (rows_cap == 0) return MOE_OK;
  if (!row_addr || !n_rows || !y_perm || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  const int64_t row_bytes = (int64_t)cfg->d_model * (cfg->x_dtype == MOE_DTYPE_BF16 ? 2 : 4);
  return from_cuda(launch_ep_peer_pull(row_bytes, n_rows, rows_cap, row_addr, y_perm,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_combine_peer(const moe_config_t* cfg, const uint64_t* row_addr, const int32_t* row_of_slot,
                     const float* topk_w, const void* shared_out, const float* shared_w, void* y, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!row_addr || !row_of_slot || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || (shared_out && !aligned16(shared_out))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_combine(*cfg, nullptr, row_of_slot, topk_w, shared_out, shared_w, y,
                                  static_cast<cudaStream_t>(stream), row_addr));
}

int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* row_of_slot,
                const float* topk_w, const void* shared_out, const float* shared_w, void* y,
                void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!row_of_slot || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || (y_perm && !aligned16(y_perm)) || (shared_out && !aligned16(shared_out)))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_combine(*cfg, y_perm, row_of_slot, topk_w, shared_out, shared_w, y,
                                  static_cast<cudaStream_t>(stream)));
}

int moe_router_stats(const moe_config_t* cfg, const int32_t* counts, const int32_t* offsets,
                     const float* p_partial, const float* lse, const int32_t* n_dropped,
                     const float* margin, float near_tie, const float* bias, float alpha, float z_coef,
                     moe_stats_t* stats, float* f_out, float* p_out, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !n_dropped || !stats) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!p_partial || !lse)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_stats(*cfg, 0, counts, offsets, p_partial, route_nblk(*cfg), lse, n_dropped, margin,
                                near_tie, nullptr, nullptr, bias, alpha, z_coef, stats, f_out, p_out, nullptr,
                                static_cast<cudaStream_t>(stream)));
}

int moe_router_stats_partial(const moe_config_t* cfg, const int32_t* counts, const int32_t* offsets,
                             const float* p_partial, const float* lse, const int32_t* n_dropped,
                             const float* margin, float near_tie, double* partial, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !n_dropped || !partial) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!p_partial || !lse)) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(partial) & 7u) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_stats(*cfg, 1, counts, offsets, p_partial, route_nblk(*cfg), lse, n_dropped, margin,
                                near_tie, nullptr, partial, nullptr, 0.f, 0.f, nullptr, nullptr, nullptr,
                                nullptr, static_cast<cudaStream_t>(stream)));
}

int moe_router_stats_finalize(const moe_config_t* cfg, const double* partial, const float* bias,
                              float alpha, float z_coef, moe_stats_t* stats, float* f_out, float* p_out,
                              int32_t* counts_out, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!partial || !stats || (reinterpret_cast<uintptr_t>(partial) & 7u)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_stats(*cfg, 2, nullptr, nullptr, nullptr, 0, nullptr, nullptr, nullptr, 0.f, partial,
                                nullptr, bias, alpha, z_coef, stats, f_out, p_out, counts_out,
                                static_cast<cudaStream_t>(stream)));
}

int moe_bias_update(const moe_config_t* cfg, const int32_t* counts, float* bias, float rate,
                    float clamp, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !bias) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_bias_update(*cfg, counts, bias, rate, clamp, static_cast<cudaStream_t>(stream)));
}

int moe_bias_update_ema(const moe_config_t* cfg, const int32_t* counts, float* ema, float beta,
                        float* bias, float rate, float clamp, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !ema || !bias || !(beta >= 0.f && beta < 1.f)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_bias_update_ema(*cfg, counts, ema, beta, bias, rate, clamp,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_bias_update_seq(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* seq_offsets,
                        int32_t n_seq, float* bias, float rate, float clamp, void* ws,
                        size_t ws_bytes, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (n_seq < 0 || !seq_offsets || !bias || (n_seq > 0 && !topk_idx)) return MOE_ERR_INVALID_ARG;
  const size_t need = (size_t)8 * (size_t)(n_seq > 0 ? n_seq : 1) * (size_t)cfg->n_experts;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 7u)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_bias_update_seq(*cfg, topk_idx, seq_offsets, n_seq, bias, rate, clamp,
                                          static_cast<double*>(ws), static_cast<cudaStream_t>(stream)));
}

int moe_route_scores(const moe_config_t* cfg, const void* x, const float* w_gate,
                     const float* logit_offset, float* scores, float* lse, float* p_partial, void* ws,
                     size_t ws_bytes, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->shared_sink) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_gate || !scores || !lse || !p_partial) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID_ARG;
  const size_t need = route_workspace_bytes(*cfg);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (!ws || !aligned16(ws))) return MOE_ERR_INVALID_ARG;
  moe_config_t c = *cfg;
  c.n_groups = 1;
  return from_cuda(launch_route(c, x, w_gate, logit_offset, nullptr, nullptr, nullptr, lse, p_partial,
                                nullptr, nullptr, ws, static_cast<cudaStream_t>(stream), scores));
}

int moe_expert_choice_capacity(const moe_config_t* cfg, int32_t* capacity) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!capacity || !(cfg->capacity_factor > 0.0)) return MOE_ERR_INVALID_ARG;
  const double c = ceil((cfg->capacity_factor * (double)cfg->top_k * (double)cfg->T) / (double)cfg->n_experts);
  const double C = c < (double)cfg->T ? c : (double)cfg->T;
  if (C > (double)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  *capacity = (int32_t)C;
  return MOE_OK;
}

int moe_expert_choice(const moe_config_t* cfg, const void* x, const float* scores, int32_t capacity,
                      int32_t* row_of, int32_t* token_of_row, int32_t* offsets, void* x_perm,
                      int32_t* n_unpicked, void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (capacity < 0 || (int64_t)capacity > cfg->T) return MOE_ERR_INVALID_ARG;
  if ((int64_t)capacity * cfg->n_experts > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!scores || !row_of || !offsets || (capacity > 0 && (!token_of_row || !x_perm || !x)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return MOE_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || (x_perm && !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_expert_choice(*cfg, x, scores, capacity, row_of, token_of_row, offsets, x_perm,
                                        n_unpicked, static_cast<cudaStream_t>(stream)));
}

int moe_combine_ec(const moe_config_t* cfg, const void* y_perm, const int32_t* row_of,
                   const float* scores, const void* shared_out, void* y, int32_t* n_unpicked,
                   void* stream) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!row_of || !scores || !y || !y_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(y_perm) || (shared_out && !aligned16(shared_out)))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_combine_ec(*cfg, y_perm, row_of, scores, shared_out, y, n_unpicked,
                                     static_cast<cudaStream_t>(stream)));
}

int moe_selftest_wait_timeout(int64_t limit_cycles, int32_t* completed, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > kWaitLimitCycles) return MOE_ERR_INVALID_ARG;
  capi::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles,
                                                                                      completed);
  return from_cuda(cudaGetLastError());
}

int moe_device_status(int32_t* status, int32_t reset) {
  if (!status) return MOE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  if (reset) {
    const int32_t z = 0;
    if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(z)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  *status = v;
  return MOE_OK;
}

int moe_last_cuda_error(void) { return (int)g_last_cuda_error; }

const char* moe_last_cuda_error_string(void) { return cudaGetErrorName(g_last_cuda_error); }

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
