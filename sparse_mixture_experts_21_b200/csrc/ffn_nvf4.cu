// NVFP4 expert compute (the MoE common-taste page, §2 table, names NVFP4 expert
// compute beside FP8 / MXFP8).  Reading of the format (NVIDIA's two-level NVFP4):
// E2M1 codes (1 sign, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes 0,
// 0.5, 1, 1.5, 2, 3, 4, 6), one unsigned E4M3 scale b per 16 consecutive elements of
// the contraction dimension and one fp32 scale g per tensor.  In fp32 and in this
// order: b = E4M3(amax_16 / fp32(6 g)) (nearest even, saturating at 448),
// s = fp32(b g), code = E2M1(fp32(x / s)) (nearest even, saturating at 6); a block
// with b = 0 is all zero codes.  Weights take g = amax / (6 * 448) per expert
// matrix; activations (the permuted x rows and h) take g = 1.
//
// Codes are packed two per byte (element 2i in the low nibble).  Scales are stored
// in GEMM-tile order ("tile atoms", as for MXFP8): rows are cut into tiles of 128
// (per group for grouped rows, tiles numbered in group order); the scales of tile t
// and 64-wide K chunk c form the 512-byte atom at (t * (cols / 64) + c) * 512, in
// which scale j (elements 64 c + 16 j ..) of the tile's row m sits at byte
// 16 (m % 32) + 4 (m / 32) + j -- the arrangement tcgen05.cp 32x128b.warpx4 moves
// into TMEM, one atom per K = 64 MMA.
//
//   nv_amax / nv_tensor_scale  per-tensor amax, then g (weights, once)
//   nv_quant_rows              bf16 [R, C] -> codes [R, C / 2] + atoms
//   nv_quant_scatter           the permutation's quantising scatter (each token's
//                              row quantised once, written to all its kept rows and,
//                              for the shared experts, to token order)
//   ffn_nv                     grouped SwiGLU FFN on tcgen05.mma.kind::mxf4nvf4
//                              .block_scale.scale_vec::4X: the tensor cores apply the
//                              E4M3 block scales inside the MMA; the epilogue applies
//                              the weights' tensor scales, SwiGLU, and re-quantises h
//                              (pass 0) or writes bf16 y (pass 1).
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace nv {

constexpr float kE2M1Max = 6.0f;
constexpr float kTensorDiv = 6.0f * 448.0f;     // g = amax / (6 * 448)

// E4M3 (nearest even, saturating) of a non-negative fp32 value, as a byte.
__device__ __forceinline__ uint32_t e4m3_byte(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Value of a non-negative E4M3 byte (sign bit clear): from the format, exactly.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return (float)m * (1.0f / 512.0f);                 // m 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));        // (1 + m/8) 2^(e-7)
}

// Two fp32 values -> one byte of E2M1 codes (lo in bits 0..3), nearest even,
// saturating at +-6.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Byte of scale j of row m (0..127) of tile `tile`, 64-wide K chunk c.
__device__ __forceinline__ int64_t atom_byte(int64_t tile, int nchunk, int c, int m, int j) {
  return (tile * nchunk + c) * 512 + 16 * (m & 31) + 4 * (m >> 5) + j;
}

// Quantise 8 consecutive elements of one 16-element block (the other 8 are in the
// neighbouring lane, lane ^ 1) with tensor scale g: 4 code bytes packed in a word,
// and the block's scale byte.
__device__ __forceinline__ uint32_t quant8(const float* f, float g, uint32_t* bscale) {
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(f[u]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  const uint32_t b = e4m3_byte(__fdiv_rn(amax, __fmul_rn(kE2M1Max, g)));
  *bscale = b;
  if (b == 0) return 0u;
  const float s = __fmul_rn(e4m3_value(b), g);
  uint32_t w = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) w |= e2m1x2(__fdiv_rn(f[2 * u], s), __fdiv_rn(f[2 * u + 1], s)) << (8 * u);
  return w;
}

// ---------------------------------------------------------------- tensor scales
// amax of each tensor of `tensor_rows` rows into bits[t] (fp32 bit patterns of
// non-negative values order like the values; bits must start at 0).
__global__ void __launch_bounds__(256)
nv_amax_kernel(const uint4* __restrict__ x, int64_t rows, int cols, int tensor_rows, uint32_t* __restrict__ bits) {
  const int64_t n8 = rows * (int64_t)cols / 8;
  const int64_t per_t = (int64_t)tensor_rows * cols / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  // warp-uniform loop: the whole warp takes 32 consecutive 8-element pieces
  for (int64_t base = warp0 * 32; base < n8; base += nwarps * 32) {
    const int64_t i = base + lane;
    const bool ok = i < n8;
    float a = 0.f;
    if (ok) {
      float f[8];
      unpack16(ldg_nc16(x + i), f, __nv_bfloat16());
#pragma unroll
      for (int u = 0; u < 8; ++u) a = fmaxf(a, fabsf(f[u]));
    }
    // one atomic per warp when its pieces lie in one tensor, else one per piece
    const int64_t t = (ok ? i : base) / per_t;
    if (__all_sync(0xffffffffu, t == base / per_t)) {
      a = warp_max(a);
      if (lane == 0) atomicMax(bits + t, __float_as_uint(a));
    } else if (ok) {
      atomicMax(bits + t, __float_as_uint(a));
    }
  }
}

// g[t] = amax / (6 * 448), 1 for an all-zero tensor (in place over the amax bits).
__global__ void nv_tensor_scale_kernel(float* __restrict__ g, int n) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) {
    const float amax = g[t];
    g[t] = amax > 0.f ? __fdiv_rn(amax, kTensorDiv) : 1.0f;
  }
}

// ---------------------------------------------------------------- quantisation
// A thread owns 8 consecutive elements; 2 consecutive threads own one 16-block.
__global__ void __launch_bounds__(256)
nv_quant_rows_kernel(const uint4* __restrict__ x, int64_t rows, int cols, int tensor_rows,
                     const float* __restrict__ g, uint32_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int64_t n8 = rows * (int64_t)cols / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t base = warp0 * 32; base < n8; base += nwarps * 32) {
    const int64_t i = base + lane;
    const bool ok = i < n8;
    float f[8];
    if (ok) unpack16(ldg_nc16(x + i), f, __nv_bfloat16());
    else {
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] = 0.f;
    }
    const int64_t r = (i * 8) / cols;
    const int c = (int)((i * 8) % cols);
    const float gt = (tensor_rows > 0 && ok) ? g[r / tensor_rows] : 1.0f;
    uint32_t b;
    const uint32_t w = quant8(f, gt, &b);
    if (ok) {
      q[i] = w;
      if ((lane & 1) == 0) sf[atom_byte(r >> 7, cols / 64, c / 64, (int)(r & 127), (c / 16) & 3)] = (uint8_t)b;
    }
  }
}

// One warp per token; per step a warp covers 256 columns (8 per lane, a 16-block per
// lane pair).  The tile of a kept row r of expert e is tp[e] + (r - offsets[e]) / 128,
// tp = exclusive scan of the experts' tile counts (recomputed per block in shared
// memory).  Activations take tensor scale 1.
constexpr int kScatterMaxN = 1024;

__global__ void __launch_bounds__(256)
nv_quant_scatter_kernel(const uint4* __restrict__ x, int64_t T, int k, int d, int N,
                        const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ row_of_slot,
                        const int32_t* __restrict__ offsets, uint8_t* __restrict__ q_perm,
                        uint8_t* __restrict__ sf_perm, uint8_t* __restrict__ q_tok,
                        uint8_t* __restrict__ sf_tok) {
  __shared__ int32_t tp[kScatterMaxN];
  __shared__ int32_t off[kScatterMaxN];
  const int lane = threadIdx.x & 31, warp_in = threadIdx.x >> 5;
  if (row_of_slot) {
    for (int e = threadIdx.x; e < N; e += blockDim.x) off[e] = offsets[e];
    if (warp_in == 0) {
      int carry = 0;
      for (int base = 0; base < N; base += 32) {
        const int e = base + lane;
        int n = 0;
        if (e < N) n = (offsets[e + 1] - offsets[e] + 127) / 128;
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < N) tp[e] = carry + incl - n;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
  __syncthreads();
  const int nchunk = d / 64;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = warp0; t < T; t += nwarps) {
    // lane j < k: the tile and the row within it of slot j (tile -1: dropped)
    int64_t my_tile = -1;
    int my_m = 0;
    int32_t my_row = -1;
    if (row_of_slot && lane < k) {
      my_row = row_of_slot[t * k + lane];
      const int e = my_row >= 0 ? topk_idx[t * k + lane] : -1;
      if ((unsigned)e >= (unsigned)N && my_row >= 0) {
        flag_invalid_index();           // a kept slot with an expert id outside [0, N)
        my_row = -1;
      }
      if (my_row >= 0) {
        const int within = my_row - off[e];
        my_tile = tp[e] + within / 128;
        my_m = within & 127;
      }
    }
    const uint4* src = x + t * (d / 8);
    for (int c0 = 0; c0 < d; c0 += 256) {
      const int col = c0 + 8 * lane;
      const bool ok = col < d;                      // uniform over each lane pair (d % 16 == 0)
      float f[8];
      if (ok) unpack16(ldg_nc16(src + col / 8), f, __nv_bfloat16());
      else {
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = 0.f;
      }
      uint32_t b;
      const uint32_t code = quant8(f, 1.0f, &b);
      const bool sf_lane = ok && (lane & 1) == 0;
      const int j = (col / 16) & 3;
      if (q_tok && ok) {
        *reinterpret_cast<uint32_t*>(q_tok + t * (d / 2) + col / 2) = code;
        if (sf_lane) sf_tok[atom_byte(t >> 7, nchunk, col / 64, (int)(t & 127), j)] = (uint8_t)b;
      }
      for (int s = 0; s < k && row_of_slot; ++s) {
        const int32_t row = __shfl_sync(0xffffffffu, my_row, s);
        const int64_t tile = __shfl_sync(0xffffffffu, my_tile, s);
        const int m = __shfl_sync(0xffffffffu, my_m, s);
        if (row < 0) continue;
        if (ok) {
          *reinterpret_cast<uint32_t*>(q_perm + (int64_t)row * (d / 2) + col / 2) = code;
          if (sf_lane) sf_perm[atom_byte(tile, nchunk, col / 64, m, j)] = (uint8_t)b;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- grouped GEMM
// One stage = 256 elements of K = 128 bytes of codes per row: A 16 KB, B 32 KB, and
// twelve scale atoms (A: four chunks; B: two 128-row tiles x four chunks).
constexpr int BM = 128, BKB = 128, BKE = 256, STAGES = 3;
constexpr int A_BYTES = BM * BKB;                // 16 KB
constexpr int B_BYTES = 256 * BKB;               // 32 KB
constexpr int ATOM = 512;
constexpr int SF_BYTES = 12 * ATOM;              // A 4 atoms, B0 4 atoms, B1 4 atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // TMA bytes of codes per stage
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int kMaxGroups = 512;
constexpr uint32_t kSfCol0 = 256;                // TMEM: accumulator [0, 256), scales after
constexpr uint32_t kSfColsPerStage = 48;         // A atoms at +4c, B of MMA c at +16 + 8c (tile 0, tile 1)

struct __align__(128) NvShared {
  uint8_t sf[STAGES][SF_BYTES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull;
  uint64_t tempty;
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  int32_t goff[kMaxGroups + 1];
  int32_t tpre[kMaxGroups + 1];
};

// The down pass stages its bf16 output through shared memory for TMA stores: one
// 32-row x 32-column box (2 KB, 64-byte swizzle) per epilogue warp.
constexpr int OUT_BOX = 2048;
constexpr size_t kSharedPad = (sizeof(NvShared) + 1023) / 1024 * 1024;
constexpr size_t kSmem = 1024 + (size_t)STAGES * STAGE_BYTES + kSharedPad + (size_t)EPI_WARPS * OUT_BOX;
static_assert(kSmem <= 227 * 1024, "shared memory of the NVFP4 GEMM");

__device__ __forceinline__ bool waitnv(uint64_t* bar, uint32_t parity, NvShared* sh) {
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

struct Tile {
  int g, row0, rows, n0, tile;   // tile: index of the 128-row tile in group-tile order
};

__device__ __forceinline__ Tile decode(int L, const NvShared* sh, int G, int tiles_n, int BN) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh->tpre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int local = L - sh->tpre[g] * tiles_n;
  const int mt = sh->tpre[g + 1] - sh->tpre[g];
  const int n_tile = local / mt, m_tile = local - n_tile * mt;
  Tile t;
  t.g = g;
  t.row0 = sh->goff[g] + m_tile * BM;
  t.rows = min(BM, sh->goff[g + 1] - t.row0);
  t.n0 = n_tile * BN;
  t.tile = sh->tpre[g] + m_tile;
  return t;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::mxf4nvf4 with block scaling: E2M1 x E2M1, UE4M3
// scales (one per 16 elements: scale_vec::4X, scale ids 0), both operands K-major,
// K = 64 per instruction.
__host__ __device__ constexpr uint32_t idesc_nv(int M, int N) {
  return (1u << 7)                            // A format E2M1
         | (1u << 10)                         // B format E2M1
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16; scale type bit 23 = 0: UE4M3
}

__device__ __forceinline__ void umma_nv(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of a 32-row x 16-byte block without swizzle (8-row core
// matrices of 128 contiguous bytes): one scale atom.
__device__ __forceinline__ uint64_t sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;           // leading byte offset
  d |= (uint64_t)(128u >> 4) << 32;           // stride byte offset: 8 rows x 16 B
  d |= (uint64_t)1u << 46;                    // descriptor version (sm_100)
  return d;                                   // layout type 0: no swizzle
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

// MODE 0: A = x codes [rows_cap, K / 2], B0 / B1 = W1 / W3 codes [G f, K / 2] with
//         tensor scales gb0 / gb1 [G]; writes h codes [rows_cap, f / 2] and h atoms.
// MODE 1: A = h codes [rows_cap, K / 2], B0 = W2 codes [G d, K / 2] with tensor
//         scales gb0 [G]; writes y bf16 [rows_cap, d].
// Tiles of 128 rows of one group x BN output columns, taken round-robin (every tile
// has the same length); a group's last tile computes on whatever rows follow and
// stores only its own.  Warp roles: 0 = producer (TMA codes + bulk-copied scale
// atoms), 1 = TMEM allocator + MMA issuer (tcgen05.cp of the atoms, four K = 64
// block-scaled MMAs per stage), 2..9 = epilogue.  Every wait is bounded; on timeout
// the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees
// TMEM and returns.
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
ffn_nv_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const uint8_t* __restrict__ sfa,
              const uint8_t* __restrict__ sfb0, const uint8_t* __restrict__ sfb1,
              const float* __restrict__ gb0, const float* __restrict__ gb1,
              const int32_t* __restrict__ offsets, int G, int K, int n_out, int64_t rows_cap,
              uint8_t* __restrict__ out_q, uint8_t* __restrict__ out_sf, __nv_bfloat16* __restrict__ out,
              const __grid_constant__ CUtensorMap tmY) {
  constexpr int BN = MODE == 0 ? 128 : 256;      // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  NvShared* sh = reinterpret_cast<NvShared*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = K / BKE;
  const int nchunk = K / 64;
  const int64_t b_tiles = (int64_t)G * n_out / 128;      // 128-row tiles of B

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
    mbar_init(&sh->tfull, 1);
    mbar_init(&sh->tempty, EPI_WARPS);
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
    // ---------------- producer (one thread)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile t = decode(L, sh, G, tiles_n, BN);
        const int64_t brow = (int64_t)t.g * n_out + t.n0;
        const int64_t bt0 = brow / 128;
        // MODE 1: the second B tile is the next 128 rows (past the end: repeat the first;
        // those output columns are not stored)
        const int64_t bt1 = MODE == 0 ? bt0 : (bt0 + 1 < b_tiles ? bt0 + 1 : bt0);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!waitnv(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          uint8_t* sfs = sh->sf[stage];
          mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES + SF_BYTES);
          tma_load_2d(&tmA, a, &sh->full[stage], kb * BKB, t.row0);
          tma_load_2d(&tmB0, b, &sh->full[stage], kb * BKB, (int32_t)brow);
          if (MODE == 0) tma_load_2d(&tmB1, b + B_BYTES / 2, &sh->full[stage], kb * BKB, (int32_t)brow);
          bulk_load(sfs, sfa + ((int64_t)t.tile * nchunk + 4 * kb) * ATOM, 4 * ATOM, &sh->full[stage]);
          bulk_load(sfs + 4 * ATOM, sfb0 + (bt0 * nchunk + 4 * kb) * ATOM, 4 * ATOM, &sh->full[stage]);
          bulk_load(sfs + 8 * ATOM, (MODE == 0 ? sfb1 : sfb0) + (bt1 * nchunk + 4 * kb) * ATOM, 4 * ATOM,
                    &sh->full[stage]);
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
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nv(BM, 256);
      uint32_t stage = 0, phase = 0, tile_i = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tile_i) {
        if (!waitnv(&sh->tempty, (tile_i & 1u) ^ 1u, sh)) { ok = false; break; }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!waitnv(&sh->full[stage], phase, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          const uint32_t sf_addr = smem_u32(sh->sf[stage]);
          const uint32_t sfa_t = tmem_base + kSfCol0 + stage * kSfColsPerStage;
          const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tmem_cp_sf(sfa_t + 4 * c, sf_desc(sf_addr + c * ATOM));
            tmem_cp_sf(sfb_t + 8 * c, sf_desc(sf_addr + (4 + c) * ATOM));
            tmem_cp_sf(sfb_t + 8 * c + 4, sf_desc(sf_addr + (8 + c) * ATOM));
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            umma_nv(tmem_base, umma_desc_sw128(a_addr + c * 32), umma_desc_sw128(b_addr + c * 32), idesc,
                    sfa_t + 4 * c, sfb_t + 8 * c, (kb | c) != 0 ? 1u : 0u);
          umma_commit(&sh->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&sh->tfull);
      }
      umma_commit(&sh->mma_done);
      mbar_wait(&sh->mma_done, 0);
    }
  } else {
    // ---------------- epilogue: TMEM lanes 32 q .. 32 q + 31; MODE 0: gate columns
    // c_lo .. c_lo + 63 and up columns 128 + c_lo ..; MODE 1: output columns c_lo .. + 127
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int c_lo = MODE == 0 ? half * 64 : half * 128;
    // down pass: this warp's output staging box (1024-aligned, for the 64-byte swizzle)
    const uint32_t box = smem_u32(smem + (size_t)STAGES * STAGE_BYTES + kSharedPad) + (warp - 2) * OUT_BOX;
    bool box_busy = false;                    // a TMA store may still be reading the box
    uint32_t tile_i = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tile_i) {
      const Tile t = decode(L, sh, G, tiles_n, BN);
      if (!waitnv(&sh->tfull, tile_i & 1u, sh)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16);
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 128; c += 16) {
        const int col = MODE == 0 ? (c < 64 ? c_lo + c : 128 + c_lo + c - 64) : c_lo + c;
        tmem_ld16(tb + col, v + c);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->tempty);        // accumulator free for the next tile
      if (MODE == 1 && q * 32 + 32 <= t.rows && t.n0 + c_lo < n_out) {
        // all 32 rows of this warp are the group's: four 32 x 32 boxes through shared
        // memory (lane l writes row l's 64 bytes, 16-byte chunk c at slot c ^ ((l >> 1) & 3),
        // the 64-byte swizzle), fenced for the TMA engine, stored by lane 0; the store
        // clips columns past the output.  A group's last, partial tile stores row by row.
        const float s2 = gb0[t.g];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (box_busy) {
            if (lane == 0) bulk_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = __fmul_rn(__uint_as_float(v[cc * 32 + c * 8 + i]), s2);
            sts16(box + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), pack16(o, __nv_bfloat16()));
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, box, t.n0 + c_lo + cc * 32, t.row0 + q * 32);
            bulk_commit();
          }
          box_busy = true;
        }
        continue;
      }
      const int r = q * 32 + lane;
      const int64_t grow = (int64_t)t.row0 + r;
      if (r >= t.rows || grow >= rows_cap) continue;
      if (MODE == 0) {
        // h = silu(g1 gate) * (g3 up) for 64 hidden units, then NVFP4 (tensor scale 1)
        // in four blocks of 16: one 32-byte run of codes and one word of scales
        const float s1 = gb0[t.g], s3 = gb1[t.g];
        uint8_t* dq = out_q + grow * (int64_t)(n_out / 2) + (t.n0 + c_lo) / 2;
        uint32_t sfw = 0, w[8];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          float h[16];
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            h[j] = silu(__fmul_rn(__uint_as_float(v[16 * blk + j]), s1)) *
                   __fmul_rn(__uint_as_float(v[64 + 16 * blk + j]), s3);
            amax = fmaxf(amax, fabsf(h[j]));
          }
          const uint32_t b = e4m3_byte(__fdiv_rn(amax, kE2M1Max));
          sfw |= b << (8 * blk);
          const float s = e4m3_value(b);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            uint32_t word = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int j = 8 * u + 2 * p;
              if (b != 0) word |= e2m1x2(__fdiv_rn(h[j], s), __fdiv_rn(h[j + 1], s)) << (8 * p);
            }
            w[2 * blk + u] = word;
          }
        }
        *reinterpret_cast<uint4*>(dq) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(dq + 16) = make_uint4(w[4], w[5], w[6], w[7]);
        // the four scales of row r in the atom of (this tile, K chunk (n0 + c_lo) / 64) of h
        *reinterpret_cast<uint32_t*>(out_sf + atom_byte(t.tile, n_out / 64, (t.n0 + c_lo) / 64, r, 0)) = sfw;
      } else if (t.n0 + c_lo < n_out) {
        const float s2 = gb0[t.g];
        __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0 + c_lo;
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          float o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = __fmul_rn(__uint_as_float(v[j + i]), s2);
          stg16(orow + j, pack16(o, __nv_bfloat16()));
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
cudaError_t launch_nv(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const uint8_t* sfa,
                      const uint8_t* sfb0, const uint8_t* sfb1, const float* gb0, const float* gb1,
                      const int32_t* offsets, int G, int K, int n_out, int64_t rows_cap, uint8_t* out_q,
                      uint8_t* out_sf, void* out, cudaStream_t s) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  const cudaError_t e = ensure_smem_attr((const void*)ffn_nv_kernel<MODE>, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + BM - 1) / BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  // the down pass's output map (the gate/up pass writes no bf16 rows and never reads it)
  CUtensorMap my{};
  if (MODE == 1 && !make_map_bf16_store32(&my, out, (uint64_t)rows_cap, (uint64_t)n_out))
    return cudaErrorInvalidValue;
  ffn_nv_kernel<MODE><<<grid, THREADS, kSmem, s>>>(a, b0, b1, sfa, sfb0, sfb1, gb0, gb1, offsets, G, K, n_out,
                                                   rows_cap, out_q, out_sf, static_cast<__nv_bfloat16*>(out), my);
  return cudaGetLastError();
}

}  // namespace nv

cudaError_t launch_nv_quant_rows(const void* x, int64_t rows, int cols, int tensor_rows, uint8_t* q, uint8_t* sf,
                                 float* g, cudaStream_t s) {
  const int64_t n8 = rows * (int64_t)cols / 8;
  if (n8 == 0) return cudaSuccess;
  const int64_t want = (n8 + 255) / 256, cap = (int64_t)sm_count() * 16;
  const int grid = (int)(want < cap ? want : cap);
  if (tensor_rows > 0) {
    const int nt = (int)(rows / tensor_rows);
    cudaError_t e = cudaMemsetAsync(g, 0, sizeof(float) * nt, s);
    if (e != cudaSuccess) return e;
    nv::nv_amax_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), rows, cols, tensor_rows,
                                            reinterpret_cast<uint32_t*>(g));
    nv::nv_tensor_scale_kernel<<<(nt + 255) / 256, 256, 0, s>>>(g, nt);
  }
  nv::nv_quant_rows_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), rows, cols, tensor_rows, g,
                                                reinterpret_cast<uint32_t*>(q), sf);
  return cudaGetLastError();
}

cudaError_t launch_nv_quant_scatter(const void* x, int64_t T, int k, int d, int N, const int32_t* topk_idx,
                                    const int32_t* row_of_slot, const int32_t* offsets, uint8_t* q_perm,
                                    uint8_t* sf_perm, uint8_t* q_tok, uint8_t* sf_tok, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (N > nv::kScatterMaxN) return cudaErrorInvalidValue;
  const int64_t want = (T + 7) / 8, cap = (int64_t)sm_count() * 8;
  nv::nv_quant_scatter_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(x), T, k, d, N, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q_tok, sf_tok);
  return cudaGetLastError();
}

cudaError_t launch_ffn_nv(const uint8_t* xq, const uint8_t* xsf, int64_t rows_cap, const int32_t* offsets, int G,
                          const uint8_t* w1q, const uint8_t* w1sf, const float* g1, const uint8_t* w3q,
                          const uint8_t* w3sf, const float* g3, const uint8_t* w2q, const uint8_t* w2sf,
                          const float* g2, int d, int f, uint8_t* hq, uint8_t* hsf, void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > nv::kMaxGroups) return cudaErrorInvalidValue;
  // code matrices are bytes: two E2M1 codes per byte, 128-byte boxes
  CUtensorMap mx, m1, m3, mh, m2;
  if (!make_map_u8(&mx, xq, rows_cap, d / 2, 128) || !make_map_u8(&m1, w1q, (uint64_t)G * f, d / 2, 128) ||
      !make_map_u8(&m3, w3q, (uint64_t)G * f, d / 2, 128) || !make_map_u8(&mh, hq, rows_cap, f / 2, 128) ||
      !make_map_u8(&m2, w2q, (uint64_t)G * d, f / 2, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = nv::launch_nv<0>(mx, m1, m3, xsf, w1sf, w3sf, g1, g3, offsets, G, d, f, rows_cap, hq, hsf,
                                   nullptr, s);
  if (e != cudaSuccess) return e;
  return nv::launch_nv<1>(mh, m2, m2, hsf, w2sf, w2sf, g2, g2, offsets, G, f, d, rows_cap, nullptr, nullptr, y, s);
}

}  // namespace moe
