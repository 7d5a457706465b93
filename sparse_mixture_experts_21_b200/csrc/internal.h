// Host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// Row-major bf16 matrix [rows, cols] as a TMA tensor map: box = 64 columns x
// box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_map_bf16_store32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols);

// Padded expert count, tokens per block and scratch of the fused router.
int route_np(int n_experts);
bool route_uses_tc(const moe_config_t& c);
int route_tokens_per_block(const moe_config_t& c);
size_t route_workspace_bytes(const moe_config_t& c);

// Exact three-way bf16 split of the router weight into ws (tensor-core router only).
cudaError_t launch_route_prepare(const moe_config_t& c, const float* w_gate, void* ws, cudaStream_t s);
// w_gate == NULL: ws already holds the split (tensor-core router only).
cudaError_t launch_route(const moe_config_t& c, const void* x, const float* w_gate,
                         const float* logit_offset, const float* bias, int32_t* topk_idx,
                         float* topk_w, float* lse, float* p_partial, float* margin,
                         float* shared_w, void* ws, cudaStream_t s, float* scores = nullptr);

// Expert-choice routing (selection + gather, and the per-token combine).
cudaError_t launch_expert_choice(const moe_config_t& c, const void* x, const float* scores, int C,
                                 int32_t* row_of, int32_t* token_of_row, int32_t* offsets, void* x_perm,
                                 int32_t* n_unpicked, cudaStream_t s);
cudaError_t launch_combine_ec(const moe_config_t& c, const void* y_perm, const int32_t* row_of,
                              const float* scores, const void* shared_out, void* y, int32_t* n_unpicked,
                              cudaStream_t s);

// Token-order capacity drop and permutation.
constexpr int kPermuteTokensPerBlock = 256;
int permute_blocks(int64_t T);
size_t permute_workspace_bytes(const moe_config_t& c);
cudaError_t launch_permute(const moe_config_t& c, int64_t capacity, const void* x,
                           const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                           int32_t* row_of_slot, int32_t* token_of_row, void* x_perm,
                           int32_t* n_dropped, int32_t* blk_counts, cudaStream_t s);

// Grouped SwiGLU FFN.
cudaError_t launch_ffn_bf16(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                            const void* w1, const void* w3, const void* w2, int d, int f,
                            void* h, void* y, cudaStream_t s);
// The same FFN plus one dense group of Ts rows (xs [Ts, d], its own ws1/ws3 [f, d],
// ws2 [d, f]) in the same two launches; h [rows_cap + Ts, f] and y [rows_cap + Ts, d]
// hold its rows after the groups' rows_cap rows.
cudaError_t launch_ffn_bf16_gate_up(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                                    const void* w1, const void* w3, int d, int f, void* h, cudaStream_t s);
cudaError_t launch_ffn_bf16_down(const void* h, int64_t rows_cap, const int32_t* offsets, int G, const void* w2,
                                 int d, int f, void* y, int Ts, const void* ws2, cudaStream_t s);
cudaError_t launch_ffn_bf16_shared(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                                   const void* w1, const void* w3, const void* w2, int d, int f, void* h, void* y,
                                   const void* xs, int Ts, const void* ws1, const void* ws3, const void* ws2,
                                   cudaStream_t s);
// The same FFN with row r of group g read from x[token_of_row[r]] (x [T, d] bf16).
cudaError_t launch_ffn_bf16_gather(const void* x, int T, const int32_t* token_of_row, int64_t rows_cap,
                                   const int32_t* offsets, int G, const void* w1, const void* w3, const void* w2,
                                   int d, int f, void* h, void* y, const void* ws1, const void* ws3,
                                   const void* ws2, cudaStream_t s);
cudaError_t launch_ffn_f32(const float* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                           const float* w1, const float* w3, const float* w2, int d, int f,
                           float* h, float* y, cudaStream_t s);

cudaError_t launch_combine(const moe_config_t& c, const void* y_perm, const int32_t* row_of_slot,
                           const float* topk_w, const void* shared_out, const float* shared_w,
                           void* y, cudaStream_t s, const uint64_t* row_addr = nullptr);
// mode 0: this batch -> stats; 1: this batch -> sufficient statistics (part_out);
// 2: sufficient statistics (part_in, possibly summed over ranks) -> stats.
cudaError_t launch_stats(const moe_config_t& c, int mode, const int32_t* counts, const int32_t* offsets,
                         const float* p_partial, int nblk, const float* lse, const int32_t* n_dropped,
                         const float* margin, float near_tie, const double* part_in, double* part_out,
                         const float* bias, float alpha, float z_coef, moe_stats_t* stats, float* f_out,
                         float* p_out, int32_t* counts_out, cudaStream_t s);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device, size).
cudaError_t ensure_smem_attr(const void* func, int bytes);
cudaError_t launch_bias_update(const moe_config_t& c, const int32_t* counts, float* bias,
                               float rate, float clamp, cudaStream_t s);
cudaError_t launch_bias_update_ema(const moe_config_t& c, const int32_t* counts, float* ema, float beta,
                                   float* bias, float rate, float clamp, cudaStream_t s);
cudaError_t launch_bias_update_seq(const moe_config_t& c, const int32_t* topk_idx,
                                   const int32_t* seq_offsets, int n_seq, float* bias, float rate,
                                   float clamp, double* ws, cudaStream_t s);

cudaError_t launch_quantize_fp8(const void* x, int64_t rows, int cols, int block_rows, uint8_t* q,
                                float* scales, cudaStream_t s);
cudaError_t launch_quant_scatter(const void* x, int64_t T, int k, int d, const int32_t* row_of_slot,
                                 uint8_t* xq_perm, float* xs_perm, uint8_t* xq_tok, float* xs_tok,
                                 cudaStream_t s);
cudaError_t launch_ffn_fp8(const uint8_t* xq, const float* xs, int64_t rows_cap, const int32_t* offsets, int G,
                           const uint8_t* w1q, const float* w1s, const uint8_t* w3q, const float* w3s,
                           const uint8_t* w2q, const float* w2s, int d, int f, uint8_t* hq, float* hs,
                           void* y, cudaStream_t s);
cudaError_t launch_mx_quant_rows(const void* x, int64_t rows, int cols, uint8_t* q, uint8_t* sf,
                                 cudaStream_t s);
cudaError_t launch_mx_quant_scatter(const void* x, int64_t T, int k, int d, int N, const int32_t* topk_idx,
                                    const int32_t* row_of_slot, const int32_t* offsets, uint8_t* q_perm,
                                    uint8_t* sf_perm, uint8_t* q_tok, uint8_t* sf_tok, cudaStream_t s);
cudaError_t launch_ffn_mx(const uint8_t* xq, const uint8_t* xsf, int64_t rows_cap, const int32_t* offsets, int G,
                          const uint8_t* w1q, const uint8_t* w1sf, const uint8_t* w3q, const uint8_t* w3sf,
                          const uint8_t* w2q, const uint8_t* w2sf, int d, int f, uint8_t* hq, uint8_t* hsf,
                          void* y, cudaStream_t s);
cudaError_t launch_nv_quant_rows(const void* x, int64_t rows, int cols, int tensor_rows, uint8_t* q, uint8_t* sf,
                                 float* g, cudaStream_t s);
cudaError_t launch_nv_quant_scatter(const void* x, int64_t T, int k, int d, int N, const int32_t* topk_idx,
                                    const int32_t* row_of_slot, const int32_t* offsets, uint8_t* q_perm,
                                    uint8_t* sf_perm, uint8_t* q_tok, uint8_t* sf_tok, cudaStream_t s);
cudaError_t launch_ffn_nv(const uint8_t* xq, const uint8_t* xsf, int64_t rows_cap, const int32_t* offsets, int G,
                          const uint8_t* w1q, const uint8_t* w1sf, const float* g1, const uint8_t* w3q,
                          const uint8_t* w3sf, const float* g3, const uint8_t* w2q, const uint8_t* w2sf,
                          const float* g2, int d, int f, uint8_t* hq, uint8_t* hsf, void* y, cudaStream_t s);
cudaError_t launch_ep_plan(const int32_t* offsets_all, int W, int rank, int N, int32_t* send_splits,
                           int32_t* recv_splits, int32_t* local_offsets, int32_t* regroup_map, int64_t recv_cap,
                           cudaStream_t s);
cudaError_t launch_rows_move(const void* src, int64_t row_bytes, const int32_t* map, const int32_t* n_rows,
                             int64_t rows_cap, int scatter, void* dst, cudaStream_t s);
cudaError_t launch_ep_peer_plan(const int32_t* offsets_round, const int32_t* offsets_own, int W, int rank, int N,
                                const uint64_t* peer_rows, int64_t row_bytes, int64_t recv_cap, uint64_t* row_addr,
                                cudaStream_t s);
cudaError_t launch_ep_peer_push(const void* x, int64_t row_bytes, int64_t T, int k, const int32_t* row_of_slot,
                                const uint64_t* row_addr, int64_t rows_cap, cudaStream_t s);
cudaError_t launch_ep_peer_pull(int64_t row_bytes, const int32_t* n_rows, int64_t rows_cap, const uint64_t* row_addr,
                                void* y_perm, cudaStream_t s);
cudaError_t peer_export(const void* ptr, uint8_t* handle, int64_t* offset);
cudaError_t peer_import(const uint8_t* handle, int64_t offset, void** ptr);
int peer_close(void* ptr);
int sm_count();

}  // namespace moe
