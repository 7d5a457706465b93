// FP8 expert compute with fine-grained block scaling (the MoE common-taste page,
// §2 table: FP8 / MXFP8 expert compute; the Practice page, "精度怎么定": FP8 training with
// fine-grained precision assignment).  Reading of the scheme: activations in 1 x 128
// blocks, weights in 128 x 128 blocks, scale = amax / 448 (fp32), code =
// E4M3(x / scale) rounded to nearest even with saturation.
//
//   quantize    block amax -> scale -> E4M3 codes (one warp per 1 x 128 block, one
//               CTA per 128 x 128 block)
//   quant_scatter  quantise each token's row once and write codes + scales to all the
//               rows the permutation gave it (replaces the bf16 row gather)
//   ffn_fp8     grouped SwiGLU FFN on tcgen05.mma.kind::f8f6f4: tiles of 128 rows x
//               256 MMA columns, one K stage = 128 = one scale block.  Each stage's
//               4 MMAs write a fresh TMEM accumulator (two buffers, alternating);
//               8 drain warps add  sa[row, kb] * sb[block, kb] * partial  into fp32
//               registers (TMEM lane quarter = warp % 4, column half = which four
//               warps).  Pass 0 applies SwiGLU and re-quantises h in 1 x 128 blocks
//               (the two warps holding a row's halves exchange their amax through
//               shared memory); pass 1 writes bf16.
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace f8 {

constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------- quantisation
// 1 x 128 blocks: one warp per (row, block), 4 elements per lane.
__global__ void __launch_bounds__(256)
quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ q,
                  float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int nbc = cols / 128;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t wblk = warp0; wblk < rows * nbc; wblk += nwarps) {
    const int64_t r = wblk / nbc;
    const int b = (int)(wblk % nbc);
    const __nv_bfloat16* src = x + r * cols + b * 128 + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(src);
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    const float s = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) packed |= (uint32_t)to_e4m3(__fdiv_rn(v[i], s)) << (8 * i);
    *reinterpret_cast<uint32_t*>(q + r * cols + b * 128 + lane * 4) = packed;
    if (lane == 0) scales[r * nbc + b] = s;
  }
}

// 128 x 128 blocks: one CTA (256 threads) per block.
__global__ void __launch_bounds__(256)
quant_blocks_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ q,
                    float* __restrict__ scales) {
  __shared__ float red[8];
  const int nbc = cols / 128;
  const int64_t br = blockIdx.x / nbc;
  const int bc = blockIdx.x % nbc;
  const int tid = threadIdx.x;
  float amax = 0.f;
  for (int i = tid; i < 128 * 128; i += 256) {
    const int64_t r = br * 128 + i / 128;
    if (r < rows) amax = fmaxf(amax, fabsf(__bfloat162float(x[r * cols + bc * 128 + i % 128])));
  }
  amax = warp_max(amax);
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
  const float s = m > 0.f ? __fdiv_rn(m, kE4M3Max) : 1.f;
  for (int i = tid; i < 128 * 128; i += 256) {
    const int64_t r = br * 128 + i / 128;
    if (r < rows) {
      const int64_t o = r * cols + bc * 128 + i % 128;
      q[o] = to_e4m3(__fdiv_rn(__bfloat162float(x[o]), s));
    }
  }
  if (tid == 0) scales[br * nbc + bc] = s;
}

// Quantise each token's row once (1 x 128 blocks) and write its codes and scales to
// every row the permutation gave it (row_of_slot[t, j] >= 0), and, when xq_tok is set,
// to row t of token-order buffers too.  One warp per token; a half-warp owns one
// 128-column block of a 256-column chunk (16 lanes x 8 values).
__global__ void __launch_bounds__(256)
quant_scatter_kernel(const uint4* __restrict__ x, int64_t T, int k, int d,
                     const int32_t* __restrict__ row_of_slot, uint8_t* __restrict__ xq_perm,
                     float* __restrict__ xs_perm, uint8_t* __restrict__ xq_tok, float* __restrict__ xs_tok) {
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int nbc = d / 128;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t my_row = (row_of_slot && lane < k) ? row_of_slot[t * k + lane] : -1;
    const uint4* src = x + t * (d / 8);
    constexpr int U = 2;                                  // 256-column chunks in flight
    for (int c0 = 0; c0 < d; c0 += 256 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int col = c0 + 256 * u + 8 * lane;
        if (col < d) v[u] = ldg_nc16(src + col / 8);
      }
      uint2 code[U];
      float scale[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int col = c0 + 256 * u + 8 * lane;
        const bool ok = col < d;                          // uniform over a half-warp
        float f[8];
        if (ok) unpack16(v[u], f, __nv_bfloat16());
        else {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = 0.f;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i >> 2] |= (uint32_t)to_e4m3(__fdiv_rn(f[i], s)) << (8 * (i & 3));
        code[u] = make_uint2(w[0], w[1]);
        scale[u] = s;
      }
      for (int j = -1; j < k; ++j) {
        int64_t row;
        uint8_t* qdst;
        float* sdst;
        if (j < 0) {
          if (!xq_tok) continue;
          row = t; qdst = xq_tok; sdst = xs_tok;
        } else {
          row = __shfl_sync(0xffffffffu, my_row, j);
          if (row < 0) continue;
          qdst = xq_perm; sdst = xs_perm;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int col = c0 + 256 * u + 8 * lane;
          if (col < d) {
            *reinterpret_cast<uint2*>(qdst + row * d + col) = code[u];
            if (hl == 0) sdst[row * nbc + col / 128] = scale[u];
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- FP8 grouped GEMM
constexpr int BM = 128, BK = 128, STAGES = 4;
constexpr int A_BYTES = BM * BK;                 // 16 KB of E4M3
constexpr int B_BYTES = 256 * BK;                // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int kMaxGroups = 512;

struct __align__(8) F8Shared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  float amax_x[4][32];                 // pass 0: half 1's row amax for half 0
  float amax_y[4][32];                 // pass 0: half 0's row amax for half 1
  int32_t goff[kMaxGroups + 1];
  int32_t tpre[kMaxGroups + 1];
};

// The down pass stages its bf16 output through shared memory for TMA stores: one
// 32-row x 32-column box (2 KB, 64-byte swizzle) per drain warp.
constexpr int OUT_BOX = 2048;
constexpr size_t kSharedPad = (sizeof(F8Shared) + 1023) / 1024 * 1024;
constexpr size_t kSmem = 1024 + (size_t)STAGES * STAGE_BYTES + kSharedPad + (size_t)EPI_WARPS * OUT_BOX;
static_assert(kSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool wait8(uint64_t* bar, uint32_t parity, F8Shared* sh) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (sh->abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      flag_timeout();
      sh->abort = 1;
      return false;
    }
  }
  return true;
}

struct T8 {
  int g, row0, rows, n0;
};

__device__ __forceinline__ T8 decode8(int L, const F8Shared* sh, int G, int tiles_n, int BN) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh->tpre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int local = L - sh->tpre[g] * tiles_n;
  const int mt = sh->tpre[g + 1] - sh->tpre[g];
  const int n_tile = local / mt, m_tile = local - n_tile * mt;
  T8 t;
  t.g = g;
  t.row0 = sh->goff[g] + m_tile * BM;
  t.rows = min(BM, sh->goff[g + 1] - t.row0);
  t.n0 = n_tile * BN;
  return t;
}

__device__ __forceinline__ float silu8(float g) { return g / (1.0f + __expf(-g)); }

// a0 += x0 * s and a1 += x1 * s as one packed two-wide fp32 FMA (each half rounds
// exactly as fma.rn.f32)
__device__ __forceinline__ void fma2(float& a0, float& a1, float x0, float x1, float s) {
  asm("{\n\t.reg .b64 acc, x, sc;\n\t"
      "mov.b64 acc, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 sc, {%4, %4};\n\t"
      "fma.rn.f32x2 acc, x, sc, acc;\n\t"
      "mov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(s));
}

// E4M3 x E4M3 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// MODE 0: A = x codes [rows_cap, d], B0/B1 = W1/W3 codes [G f, d]; writes h codes
//         [rows_cap, f] and h scales [rows_cap, f / 128].
// MODE 1: A = h codes [rows_cap, f], B0 = W2 codes [G d, f]; writes y bf16 [rows_cap, d].
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
ffn_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const float* __restrict__ sa,
               const float* __restrict__ sb0, const float* __restrict__ sb1,
               const int32_t* __restrict__ offsets, int G, int K, int n_out, int64_t rows_cap,
               uint8_t* __restrict__ out_q, float* __restrict__ out_s, __nv_bfloat16* __restrict__ out,
               const __grid_constant__ CUtensorMap tmY) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  F8Shared* sh = reinterpret_cast<F8Shared*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = K / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&sh->tfull[a], 1); mbar_init(&sh->tempty[a], EPI_WARPS); }
    mbar_init(&sh->mma_done, 1);
    sh->abort = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    if (MODE == 0) prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 2) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int mt = 0;
      if (g < G) {
        const int o0 = offsets[g], o1 = offsets[g + 1];
        sh->goff[g] = o0;
        mt = o1 > o0 ? (o1 - o0 + BM - 1) / BM : 0;
      }
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (g < G) sh->tpre[g + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { sh->tpre[0] = 0; sh->goff[G] = offsets[G]; }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh->tmem_base;
  const int total = sh->tpre[G] * tiles_n;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const T8 t = decode8(L, sh, G, tiles_n, BN);
        const int brow = t.g * n_out + t.n0;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait8(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES);
          tma_load_2d(&tmA, a, &sh->full[stage], kb * BK, t.row0);
          if (MODE == 0) {
            tma_load_2d(&tmB0, b, &sh->full[stage], kb * BK, brow);
            tma_load_2d(&tmB1, b + B_BYTES / 2, &sh->full[stage], kb * BK, brow);
          } else {
            tma_load_2d(&tmB0, b, &sh->full[stage], kb * BK, brow);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int i = 1; i <= min(issued, STAGES); ++i) {
          const int s = ((int)stage - i + 2 * STAGES) % STAGES;
          mbar_wait(&sh->full[s], ((int)stage - i < 0) ? (phase ^ 1u) : phase);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3(BM, 256);
      uint32_t stage = 0, phase = 0, gkb = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb, ++gkb) {
          const uint32_t buf = gkb & 1u;
          if (!wait8(&sh->tempty[buf], ((gkb >> 1) & 1u) ^ 1u, sh)) { ok = false; break; }
          if (!wait8(&sh->full[stage], phase, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_f8(tmem_base + buf * 256u, umma_desc_sw128(a_addr + kk * 32),
                    umma_desc_sw128(b_addr + kk * 32), idesc, kk != 0 ? 1u : 0u);
          umma_commit(&sh->empty[stage]);
          umma_commit(&sh->tfull[buf]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      umma_commit(&sh->mma_done);
      mbar_wait(&sh->mma_done, 0);
    }
  } else {
    // drain + epilogue: TMEM lanes 32 q .. 32 q + 31, 128 of the 256 columns.  After an
    // abort every warp keeps walking its tiles without waiting or touching TMEM, so the
    // two warps of a lane quarter still meet at the same named barriers.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int c_lo = MODE == 0 ? half * 64 : half * 128;
    // down pass: this warp's output staging box (1024-aligned, for the 64-byte swizzle)
    const uint32_t box = smem_u32(smem + (size_t)STAGES * STAGE_BYTES + kSharedPad) + (warp - 2) * OUT_BOX;
    bool box_busy = false;                    // a TMA store may still be reading the box
    uint32_t gkb = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const T8 t = decode8(L, sh, G, tiles_n, BN);
      const int r = q * 32 + lane;
      const int64_t grow = (int64_t)t.row0 + r;
      const bool row_ok = r < t.rows && grow < rows_cap;
      const bool col_ok = MODE == 0 || t.n0 + c_lo < n_out;
      // the weight scale block row of this thread's columns
      const int64_t blk = (int64_t)(t.g * n_out + t.n0 + (MODE == 0 ? 0 : c_lo)) / 128;
      const float* sa_row = sa + (row_ok ? grow : 0) * (int64_t)nkb;
      const float* sb0_row = sb0 + (col_ok ? blk : 0) * (int64_t)nkb;
      const float* sb1_row = MODE == 0 ? sb1 + blk * (int64_t)nkb : sb0_row;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      float a_s = sa_row[0], b0_s = sb0_row[0], b1_s = sb1_row[0];
      for (int kb = 0; kb < nkb; ++kb, ++gkb) {
        const int kn = kb + 1 < nkb ? kb + 1 : kb;            // next block's scales, loaded ahead
        const float a_n = sa_row[kn], b0_n = sb0_row[kn], b1_n = sb1_row[kn];
        const uint32_t buf = gkb & 1u;
        if (ok && !wait8(&sh->tfull[buf], (gkb >> 1) & 1u, sh)) ok = false;
        if (ok) {
          tc_fence_after();
          const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + buf * 256u;
          const float sr = (row_ok && col_ok) ? a_s : 0.f;
          const float s0 = sr * b0_s, s1 = sr * b1_s;
#pragma unroll
          for (int part = 0; part < 4; ++part) {
            // MODE 0: parts 0, 1 = gate columns c_lo + 0..63, parts 2, 3 = up columns
            // 128 + c_lo + 0..63.  MODE 1: parts 0..3 = output columns c_lo + 0..127.
            const int col = MODE == 0 ? (part < 2 ? c_lo + 32 * part : 128 + c_lo + 32 * (part - 2))
                                      : c_lo + 32 * part;
            uint32_t v[32];
            tmem_ld16(tb + col, v);
            tmem_ld16(tb + col + 16, v + 16);
            tmem_ld_wait();
            const float sc = (MODE == 0 && part >= 2) ? s1 : s0;
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              fma2(acc[32 * part + i], acc[32 * part + i + 1], __uint_as_float(v[i]), __uint_as_float(v[i + 1]), sc);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->tempty[buf]);
        }
        a_s = a_n; b0_s = b0_n; b1_s = b1_n;
      }
      if (MODE == 0) {
        // h = silu(gate) * up for this thread's 64 hidden units; a row's 128 units sit in
        // the two warps of this lane quarter, which exchange their amax
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          acc[j] = silu8(acc[j]) * acc[64 + j];
          amax = fmaxf(amax, fabsf(acc[j]));
        }
        if (half == 0) sh->amax_y[q][lane] = amax; else sh->amax_x[q][lane] = amax;
        named_bar(1 + q, 64);
        amax = fmaxf(amax, half == 0 ? sh->amax_x[q][lane] : sh->amax_y[q][lane]);
        named_bar(1 + q, 64);
        const float s = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
        if (ok && row_ok) {
          uint8_t* dq = out_q + grow * (int64_t)n_out + t.n0 + half * 64;
#pragma unroll
          for (int j = 0; j < 64; j += 16) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float* a4 = acc + j + 4 * u;
              w[u] = (uint32_t)to_e4m3(__fdiv_rn(a4[0], s)) | ((uint32_t)to_e4m3(__fdiv_rn(a4[1], s)) << 8) |
                     ((uint32_t)to_e4m3(__fdiv_rn(a4[2], s)) << 16) |
                     ((uint32_t)to_e4m3(__fdiv_rn(a4[3], s)) << 24);
            }
            *reinterpret_cast<uint4*>(dq + j) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (half == 0) out_s[grow * (int64_t)(n_out / 128) + t.n0 / 128] = s;
        }
      } else if (__all_sync(0xffffffffu, ok) && q * 32 + 32 <= t.rows && col_ok) {
        // all 32 rows of this warp are the group's: four 32 x 32 boxes through shared
        // memory (lane l writes row l's 64 bytes, 16-byte chunk c at slot c ^ ((l >> 1) & 3),
        // the 64-byte swizzle), fenced for the TMA engine, stored by lane 0; the store
        // clips columns past the output.  A group's last, partial tile stores row by row.
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (box_busy) {
            if (lane == 0) bulk_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float* e = acc + cc * 32 + c * 8;
            uint4 pk;
            pk.x = pack_bf16x2(e[0], e[1]); pk.y = pack_bf16x2(e[2], e[3]);
            pk.z = pack_bf16x2(e[4], e[5]); pk.w = pack_bf16x2(e[6], e[7]);
            sts16(box + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), pk);
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, box, t.n0 + c_lo + cc * 32, t.row0 + q * 32);
            bulk_commit();
          }
          box_busy = true;
        }
      } else if (ok && row_ok && col_ok) {
        __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0 + c_lo;
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(acc[j], acc[j + 1]); pk.y = pack_bf16x2(acc[j + 2], acc[j + 3]);
          pk.z = pack_bf16x2(acc[j + 4], acc[j + 5]); pk.w = pack_bf16x2(acc[j + 6], acc[j + 7]);
          stg16(orow + j, pk);
        }
      }
    }
    // every output box of this warp is in global memory before the kernel ends
    if (MODE == 1 && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int MODE>
cudaError_t launch_f8(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const float* sa,
                      const float* sb0, const float* sb1, const int32_t* offsets, int G, int K, int n_out,
                      int64_t rows_cap, uint8_t* out_q, float* out_s, void* out, cudaStream_t s) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  const cudaError_t e = ensure_smem_attr((const void*)ffn_fp8_kernel<MODE>, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + BM - 1) / BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  // the down pass's output map (the gate/up pass writes no bf16 rows and never reads it)
  CUtensorMap my{};
  if (MODE == 1 && !make_map_bf16_store32(&my, out, (uint64_t)rows_cap, (uint64_t)n_out))
    return cudaErrorInvalidValue;
  ffn_fp8_kernel<MODE><<<grid, THREADS, kSmem, s>>>(a, b0, b1, sa, sb0, sb1, offsets, G, K, n_out, rows_cap,
                                                    out_q, out_s, static_cast<__nv_bfloat16*>(out), my);
  return cudaGetLastError();
}

}  // namespace f8

cudaError_t launch_quantize_fp8(const void* x, int64_t rows, int cols, int block_rows, uint8_t* q,
                                float* scales, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (block_rows == 1) {
    const int64_t warps = rows * (cols / 128);
    const int64_t want = (warps + 7) / 8, cap = (int64_t)sm_count() * 16;
    f8::quant_rows_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(xb, rows, cols, q, scales);
  } else {
    const int64_t blocks = ((rows + 127) / 128) * (cols / 128);
    f8::quant_blocks_kernel<<<(unsigned)blocks, 256, 0, s>>>(xb, rows, cols, q, scales);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_scatter(const void* x, int64_t T, int k, int d, const int32_t* row_of_slot,
                                 uint8_t* xq_perm, float* xs_perm, uint8_t* xq_tok, float* xs_tok,
                                 cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int64_t want = (T + 7) / 8, cap = (int64_t)sm_count() * 8;
  f8::quant_scatter_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(x), T, k, d, row_of_slot, xq_perm, xs_perm, xq_tok, xs_tok);
  return cudaGetLastError();
}

cudaError_t launch_ffn_fp8(const uint8_t* xq, const float* xs, int64_t rows_cap, const int32_t* offsets, int G,
                           const uint8_t* w1q, const float* w1s, const uint8_t* w3q, const float* w3s,
                           const uint8_t* w2q, const float* w2s, int d, int f, uint8_t* hq, float* hs,
                           void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > f8::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mx, m1, m3, mh, m2;
  if (!make_map_u8(&mx, xq, rows_cap, d, 128) || !make_map_u8(&m1, w1q, (uint64_t)G * f, d, 128) ||
      !make_map_u8(&m3, w3q, (uint64_t)G * f, d, 128) || !make_map_u8(&mh, hq, rows_cap, f, 128) ||
      !make_map_u8(&m2, w2q, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = f8::launch_f8<0>(mx, m1, m3, xs, w1s, w3s, offsets, G, d, f, rows_cap, hq, hs, nullptr, s);
  if (e != cudaSuccess) return e;
  return f8::launch_f8<1>(mh, m2, m2, hs, w2s, w2s, offsets, G, f, d, rows_cap, nullptr, nullptr, y, s);
}

}  // namespace moe
