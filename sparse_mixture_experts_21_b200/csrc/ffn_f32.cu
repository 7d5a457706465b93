// Grouped SwiGLU expert FFN in fp32 (FMA pipes): the fp32 layer variant, where
// tensor-core TF32 would not hold a 1e-4 relative error.  Same algorithm and
// group/tile ordering as the bf16 tensor-core path; see ffn_tc.cu.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace f32 {

constexpr int BM = 32, BN = 32, KC = 32, kMaxGroups = 512;

struct F32Shared {
  float a[KC][BM + 1];
  float b0[KC][BN + 1];
  float b1[KC][BN + 1];
  int32_t goff[kMaxGroups + 1];
  int32_t tpre[kMaxGroups + 1];
};

// y = silu(A B0^T) * (A B1^T) (MODE 0) or A B0^T (MODE 1), per 32 x 32 tile.
template <int MODE>
__global__ void __launch_bounds__(256)
ffn_f32_kernel(const float* __restrict__ A, const float* __restrict__ B0,
               const float* __restrict__ B1, const int32_t* __restrict__ offsets, int G, int K,
               int n_out, int64_t rows_cap, float* __restrict__ out) {
  __shared__ F32Shared sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int mt = 0;
      if (g < G) {
        const int o0 = offsets[g], o1 = offsets[g + 1];
        sh.goff[g] = o0;
        mt = o1 > o0 ? (o1 - o0 + BM - 1) / BM : 0;
      }
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (g < G) sh.tpre[g + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { sh.tpre[0] = 0; sh.goff[G] = offsets[G]; }
  }
  __syncthreads();
  const int tiles_n = (n_out + BN - 1) / BN;
  const int total = sh.tpre[G] * tiles_n;
  const int ty = tid / 16, tx = tid % 16;
  for (int L = blockIdx.x; L < total; L += gridDim.x) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sh.tpre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int local = L - sh.tpre[g] * tiles_n;
    const int mt = sh.tpre[g + 1] - sh.tpre[g];
    const int n0 = (local / mt) * BN;
    const int row0 = sh.goff[g] + (local % mt) * BM;
    const int rows = min(BM, sh.goff[g + 1] - row0);
    float acc0[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, acc1[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    for (int k0 = 0; k0 < K; k0 += KC) {
      for (int i = tid; i < BM * KC; i += 256) {
        const int r = i / KC, c = i % KC;
        const int64_t gr = (int64_t)row0 + r;
        sh.a[c][r] = (r < rows && gr < rows_cap && k0 + c < K) ? A[gr * K + k0 + c] : 0.f;
        const int n = n0 + r;
        const bool okb = n < n_out && k0 + c < K;
        const int64_t bo = ((int64_t)g * n_out + n) * K + k0 + c;
        sh.b0[c][r] = okb ? B0[bo] : 0.f;
        if (MODE == 0) sh.b1[c][r] = okb ? B1[bo] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int c = 0; c < KC; ++c) {
        const float a0 = sh.a[c][ty * 2], a1 = sh.a[c][ty * 2 + 1];
        const float p0 = sh.b0[c][tx * 2], p1 = sh.b0[c][tx * 2 + 1];
        acc0[0][0] = fmaf(a0, p0, acc0[0][0]); acc0[0][1] = fmaf(a0, p1, acc0[0][1]);
        acc0[1][0] = fmaf(a1, p0, acc0[1][0]); acc0[1][1] = fmaf(a1, p1, acc0[1][1]);
        if (MODE == 0) {
          const float u0 = sh.b1[c][tx * 2], u1 = sh.b1[c][tx * 2 + 1];
          acc1[0][0] = fmaf(a0, u0, acc1[0][0]); acc1[0][1] = fmaf(a0, u1, acc1[0][1]);
          acc1[1][0] = fmaf(a1, u0, acc1[1][0]); acc1[1][1] = fmaf(a1, u1, acc1[1][1]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = ty * 2 + i;
      const int64_t gr = (int64_t)row0 + r;
      if (r >= rows || gr >= rows_cap) continue;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int n = n0 + tx * 2 + j;
        if (n >= n_out) continue;
        float v = acc0[i][j];
        if (MODE == 0) v = v / (1.0f + expf(-v)) * acc1[i][j];
        out[gr * n_out + n] = v;
      }
    }
  }
}

}  // namespace f32


cudaError_t launch_ffn_f32(const float* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                           const float* w1, const float* w3, const float* w2, int d, int f,
                           float* h, float* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > f32::kMaxGroups) return cudaErrorInvalidValue;
  const int64_t mt = (rows_cap + f32::BM - 1) / f32::BM + G;
  const int64_t t0 = mt * ((f + f32::BN - 1) / f32::BN), t1 = mt * ((d + f32::BN - 1) / f32::BN);
  const int cap = sm_count() * 8;
  f32::ffn_f32_kernel<0><<<(int)(t0 < cap ? t0 : cap), 256, 0, s>>>(x_rows, w1, w3, offsets, G, d, f,
                                                              rows_cap, h);
  f32::ffn_f32_kernel<1><<<(int)(t1 < cap ? t1 : cap), 256, 0, s>>>(h, w2, w2, offsets, G, f, d,
                                                              rows_cap, y);
  return cudaGetLastError();
}

}  // namespace moe
