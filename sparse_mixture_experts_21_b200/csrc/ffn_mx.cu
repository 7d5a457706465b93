// MXFP8 expert compute (the MoE common-taste page, §2 table: FP8 / MXFP8 expert
// compute).  Format: OCP Microscaling MXFP8 -- E4M3 codes, one E8M0 (power-of-two)
// scale per 32 consecutive elements along the contraction dimension, scale exponent
// e = floor(log2 amax) - 8 clamped to [-127, 127], code = E4M3(x / 2^e) saturating.
//
// Scales are stored in GEMM-tile order ("tile atoms"): an operand's rows are cut
// into tiles of 128 (per group when the rows are grouped by expert: tile i of a
// group starts at offsets[g] + 128 i, tiles numbered in group order); the scales of
// tile t and 128-wide K block kb form the 512-byte atom at (t * (cols / 128) + kb)
// * 512, in which the scale j (elements 128 kb + 32 j ..) of the tile's row m sits
// at byte 16 (m % 32) + 4 (m / 32) + j -- the arrangement tcgen05.cp 32x128b.warpx4
// moves into TMEM for the block-scaled MMA.  A GEMM stage's scales are then three
// contiguous 512-byte atoms, fetched with bulk copies next to the operand tiles.
//
//   mx_quant_rows     bf16 [R, C] -> codes [R, C] + sf [R, C / 32]
//   mx_quant_scatter  the permutation's quantising scatter (as in the fine-grained
//                     FP8 path): each token's row is quantised once and written to
//                     all its kept rows (and to token order for the shared experts)
//   ffn_mx            grouped SwiGLU FFN on tcgen05.mma.kind::mxf8f6f4.block_scale:
//                     the tensor cores apply both operands' scales inside the MMA, so
//                     one TMEM accumulator runs over the whole K range.  Per 128-wide
//                     K stage one thread issues the TMA loads of the codes and bulk
//                     copies of the stage's three scale atoms; the MMA warp copies the
//                     atoms to TMEM (tcgen05.cp 32x128b.warpx4) and issues four
//                     K = 32 MMAs selecting scale byte j.  The epilogue copies the
//                     accumulator to registers, releases it, then applies SwiGLU and
//                     re-quantises h to MXFP8 (pass 0, scales written as tile atoms)
//                     or writes bf16 y (pass 1).
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace mx {

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// E8M0 byte of a block whose largest magnitude is amax (amax >= 0, finite):
// floor(log2 amax) is the float's unbiased exponent for normal amax, so the byte
// e + 127 is the biased exponent field minus 8 (clamped at 0; zero and subnormal
// amax give byte 0, e = -127).
__device__ __forceinline__ uint32_t e8m0_of(float amax) {
  const int ef = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  return ef > 8 ? (uint32_t)(ef - 8) : 0u;
}

// 2^-e for an E8M0 byte b = e + 127 (b <= 246 for finite fp32 data): exact.
__device__ __forceinline__ float inv_scale(uint32_t b) { return __uint_as_float((254u - b) << 23); }

// Byte of scale j of row m (0..127) of tile `tile`, K block kb, in the tile-atom layout.
__device__ __forceinline__ int64_t atom_byte(int64_t tile, int nkb, int kb, int m, int j) {
  return (tile * nkb + kb) * 512 + 16 * (m & 31) + 4 * (m >> 5) + j;
}

// ---------------------------------------------------------------- quantisation
// A thread owns 8 consecutive elements; 4 consecutive threads own one 32-block.
__global__ void __launch_bounds__(256)
mx_quant_rows_kernel(const uint4* __restrict__ x, int64_t rows, int cols, uint2* __restrict__ q,
                     uint8_t* __restrict__ sf) {
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
    float amax = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(f[u]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const uint32_t b = e8m0_of(amax);
    const float m = inv_scale(b);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u >> 2] |= (uint32_t)to_e4m3(f[u] * m) << (8 * (u & 3));
    if (ok) {
      q[i] = make_uint2(w[0], w[1]);
      if ((lane & 3) == 0) {
        const int64_t r = (i * 8) / cols;
        const int c = (int)((i * 8) % cols);
        sf[atom_byte(r >> 7, cols / 128, c / 128, (int)(r & 127), (c / 32) & 3)] = (uint8_t)b;
      }
    }
  }
}

// One warp per token; per step a warp covers 256 columns (8 per lane).  The tile of a
// kept row r of expert e is tp[e] + (r - offsets[e]) / 128, tp = exclusive scan of the
// experts' tile counts (recomputed per block in shared memory).
constexpr int kScatterMaxN = 1024;

__global__ void __launch_bounds__(256)
mx_quant_scatter_kernel(const uint4* __restrict__ x, int64_t T, int k, int d, int N,
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
        if (e < N) {
          const int c = offsets[e + 1] - offsets[e];
          n = (c + 127) / 128;
        }
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
  const int nkb = d / 128;
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
      const bool ok = col < d;                      // uniform over each 4-lane block
      float f[8];
      if (ok) unpack16(ldg_nc16(src + col / 8), f, __nv_bfloat16());
      else {
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(f[u]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const uint32_t b = e8m0_of(amax);
      const float mul = inv_scale(b);
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int u = 0; u < 8; ++u) w[u >> 2] |= (uint32_t)to_e4m3(f[u] * mul) << (8 * (u & 3));
      const uint2 code = make_uint2(w[0], w[1]);
      const bool sf_lane = ok && (lane & 3) == 0;
      if (q_tok && ok) {
        *reinterpret_cast<uint2*>(q_tok + t * d + col) = code;
        if (sf_lane) sf_tok[atom_byte(t >> 7, nkb, col / 128, (int)(t & 127), (col / 32) & 3)] = (uint8_t)b;
      }
      for (int j = 0; j < k && row_of_slot; ++j) {
        const int32_t row = __shfl_sync(0xffffffffu, my_row, j);
        const int64_t tile = __shfl_sync(0xffffffffu, my_tile, j);
        const int m = __shfl_sync(0xffffffffu, my_m, j);
        if (row < 0) continue;
        if (ok) {
          *reinterpret_cast<uint2*>(q_perm + (int64_t)row * d + col) = code;
          if (sf_lane) sf_perm[atom_byte(tile, nkb, col / 128, m, (col / 32) & 3)] = (uint8_t)b;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- grouped GEMM
constexpr int BM = 128, BK = 128, STAGES = 4;
constexpr int A_BYTES = BM * BK;                 // 16 KB of E4M3
constexpr int B_BYTES = 256 * BK;                // 32 KB
constexpr int SF_BYTES = 3 * 512;                // A atom + two B atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // TMA bytes of codes per stage
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int kMaxGroups = 512;
constexpr uint32_t kSfCol0 = 256;                // TMEM: accumulator [0, 256), scales after
constexpr uint32_t kSfColsPerStage = 16;         // A at +0 (4 columns), B at +8 (8 columns)

struct __align__(16) MxShared {
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
constexpr size_t kSharedPad = (sizeof(MxShared) + 1023) / 1024 * 1024;
constexpr size_t kSmem = 1024 + (size_t)STAGES * STAGE_BYTES + kSharedPad + (size_t)EPI_WARPS * OUT_BOX;
static_assert(kSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool waitmx(uint64_t* bar, uint32_t parity, MxShared* sh) {
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

__device__ __forceinline__ Tile decode(int L, const MxShared* sh, int G, int tiles_n, int BN) {
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

// Instruction descriptor, kind::mxf8f6f4 with block scaling: E4M3 x E4M3, UE8M0
// scales, both operands K-major; sf_id picks the scale byte of each operand.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, uint32_t sf_id) {
  return (sf_id << 4)                         // B scale factor id
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | (1u << 23)                         // scale type UE8M0
         | ((uint32_t)(M >> 4) << 24)         // M / 16
         | (sf_id << 29);                     // A scale factor id
}

__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of a 32-row x 16-byte block without swizzle (8-row core
// matrices of 128 contiguous bytes).
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

// MODE 0: A = x codes [rows_cap, d], B0/B1 = W1/W3 codes [G f, d]; writes h codes
//         [rows_cap, f] and h scales [rows_cap, f / 32].
// MODE 1: A = h codes [rows_cap, f], B0 = W2 codes [G d, f]; writes y bf16 [rows_cap, d].
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
ffn_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const uint8_t* __restrict__ sfa,
              const uint8_t* __restrict__ sfb0, const uint8_t* __restrict__ sfb1,
              const int32_t* __restrict__ offsets, int G, int K, int n_out, int64_t rows_cap,
              uint8_t* __restrict__ out_q, uint8_t* __restrict__ out_sf, __nv_bfloat16* __restrict__ out,
              const __grid_constant__ CUtensorMap tmY) {
  constexpr int BN = MODE == 0 ? 128 : 256;      // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  MxShared* sh = reinterpret_cast<MxShared*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = K / BK;
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
    // ---------------- producer (one thread): codes by TMA, the stage's three scale atoms
    // by bulk copies, all completing on the stage's full barrier
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile t = decode(L, sh, G, tiles_n, BN);
        const int64_t brow = (int64_t)t.g * n_out + t.n0;
        const int64_t bt0 = brow / 128;
        // MODE 1: the second B atom is the next 128 rows (past the end: repeat the first;
        // those output columns are not stored)
        const int64_t bt1 = MODE == 0 ? bt0 : (bt0 + 1 < b_tiles ? bt0 + 1 : bt0);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!waitmx(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          uint8_t* sfs = sh->sf[stage];
          mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES + SF_BYTES);
          tma_load_2d(&tmA, a, &sh->full[stage], kb * BK, t.row0);
          if (MODE == 0) {
            tma_load_2d(&tmB0, b, &sh->full[stage], kb * BK, (int32_t)brow);
            tma_load_2d(&tmB1, b + B_BYTES / 2, &sh->full[stage], kb * BK, (int32_t)brow);
          } else {
            tma_load_2d(&tmB0, b, &sh->full[stage], kb * BK, (int32_t)brow);
          }
          bulk_load(sfs, sfa + ((int64_t)t.tile * nkb + kb) * 512, 512, &sh->full[stage]);
          bulk_load(sfs + 512, sfb0 + (bt0 * nkb + kb) * 512, 512, &sh->full[stage]);
          bulk_load(sfs + 1024, (MODE == 0 ? sfb1 : sfb0) + (bt1 * nkb + kb) * 512, 512, &sh->full[stage]);
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
      uint32_t stage = 0, phase = 0, tile_i = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tile_i) {
        if (!waitmx(&sh->tempty, (tile_i & 1u) ^ 1u, sh)) { ok = false; break; }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!waitmx(&sh->full[stage], phase, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          const uint32_t sf_addr = smem_u32(sh->sf[stage]);
          const uint32_t sfa_t = tmem_base + kSfCol0 + stage * kSfColsPerStage;
          const uint32_t sfb_t = sfa_t + 8;
          tmem_cp_sf(sfa_t, sf_desc(sf_addr));
          tmem_cp_sf(sfb_t, sf_desc(sf_addr + 512));
          tmem_cp_sf(sfb_t + 4, sf_desc(sf_addr + 1024));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_mx(tmem_base, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32),
                    idesc_mx(BM, 256, (uint32_t)kk), sfa_t, sfb_t, (kb | kk) != 0 ? 1u : 0u);
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
      if (!waitmx(&sh->tfull, tile_i & 1u, sh)) break;
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
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (box_busy) {
            if (lane == 0) bulk_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t* e = v + cc * 32 + c * 8;
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(e[0]), __uint_as_float(e[1]));
            pk.y = pack_bf16x2(__uint_as_float(e[2]), __uint_as_float(e[3]));
            pk.z = pack_bf16x2(__uint_as_float(e[4]), __uint_as_float(e[5]));
            pk.w = pack_bf16x2(__uint_as_float(e[6]), __uint_as_float(e[7]));
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
        continue;
      }
      const int r = q * 32 + lane;
      const int64_t grow = (int64_t)t.row0 + r;
      if (r >= t.rows || grow >= rows_cap) continue;
      if (MODE == 0) {
        // h = silu(gate) * up for 64 hidden units, then MXFP8 in two blocks of 32
        uint8_t* dq = out_q + grow * (int64_t)n_out + t.n0 + c_lo;
        uint32_t sfw = 0;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float h[32];
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            h[j] = silu(__uint_as_float(v[32 * blk + j])) * __uint_as_float(v[64 + 32 * blk + j]);
            amax = fmaxf(amax, fabsf(h[j]));
          }
          const uint32_t b = e8m0_of(amax);
          const float m = inv_scale(b);
          sfw |= b << (8 * blk);
#pragma unroll
          for (int j0 = 0; j0 < 32; j0 += 16) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              w[u] = (uint32_t)to_e4m3(h[j0 + 4 * u] * m) | ((uint32_t)to_e4m3(h[j0 + 4 * u + 1] * m) << 8) |
                     ((uint32_t)to_e4m3(h[j0 + 4 * u + 2] * m) << 16) |
                     ((uint32_t)to_e4m3(h[j0 + 4 * u + 3] * m) << 24);
            *reinterpret_cast<uint4*>(dq + 32 * blk + j0) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        // scales c_lo / 32 and + 1 of row r in the atom of (this tile, K block n0 / 128) of h
        *reinterpret_cast<uint16_t*>(out_sf + atom_byte(t.tile, n_out / 128, t.n0 / 128, r, c_lo / 32)) =
            (uint16_t)sfw;
      } else if (t.n0 + c_lo < n_out) {
        __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0 + c_lo;
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
          pk.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
          pk.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
          pk.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
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
cudaError_t launch_mx(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const uint8_t* sfa,
                      const uint8_t* sfb0, const uint8_t* sfb1, const int32_t* offsets, int G, int K, int n_out,
                      int64_t rows_cap, uint8_t* out_q, uint8_t* out_sf, void* out, cudaStream_t s) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  const cudaError_t e = ensure_smem_attr((const void*)ffn_mx_kernel<MODE>, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + BM - 1) / BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  // the down pass's output map (the gate/up pass writes no bf16 rows and never reads it)
  CUtensorMap my{};
  if (MODE == 1 && !make_map_bf16_store32(&my, out, (uint64_t)rows_cap, (uint64_t)n_out))
    return cudaErrorInvalidValue;
  ffn_mx_kernel<MODE><<<grid, THREADS, kSmem, s>>>(a, b0, b1, sfa, sfb0, sfb1, offsets, G, K, n_out, rows_cap,
                                                   out_q, out_sf, static_cast<__nv_bfloat16*>(out), my);
  return cudaGetLastError();
}

}  // namespace mx

cudaError_t launch_mx_quant_rows(const void* x, int64_t rows, int cols, uint8_t* q, uint8_t* sf,
                                 cudaStream_t s) {
  const int64_t n8 = rows * (int64_t)cols / 8;
  if (n8 == 0) return cudaSuccess;
  const int64_t want = (n8 + 255) / 256, cap = (int64_t)sm_count() * 16;
  mx::mx_quant_rows_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(x), rows, cols, reinterpret_cast<uint2*>(q), sf);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_scatter(const void* x, int64_t T, int k, int d, int N, const int32_t* topk_idx,
                                    const int32_t* row_of_slot, const int32_t* offsets, uint8_t* q_perm,
                                    uint8_t* sf_perm, uint8_t* q_tok, uint8_t* sf_tok, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (N > mx::kScatterMaxN) return cudaErrorInvalidValue;
  const int64_t want = (T + 7) / 8, cap = (int64_t)sm_count() * 8;
  mx::mx_quant_scatter_kernel<<<(int)(want < cap ? want : cap), 256, 0, s>>>(
      static_cast<const uint4*>(x), T, k, d, N, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q_tok, sf_tok);
  return cudaGetLastError();
}

cudaError_t launch_ffn_mx(const uint8_t* xq, const uint8_t* xsf, int64_t rows_cap, const int32_t* offsets, int G,
                          const uint8_t* w1q, const uint8_t* w1sf, const uint8_t* w3q, const uint8_t* w3sf,
                          const uint8_t* w2q, const uint8_t* w2sf, int d, int f, uint8_t* hq, uint8_t* hsf,
                          void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > mx::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mxm, m1, m3, mh, m2;
  if (!make_map_u8(&mxm, xq, rows_cap, d, 128) || !make_map_u8(&m1, w1q, (uint64_t)G * f, d, 128) ||
      !make_map_u8(&m3, w3q, (uint64_t)G * f, d, 128) || !make_map_u8(&mh, hq, rows_cap, f, 128) ||
      !make_map_u8(&m2, w2q, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = mx::launch_mx<0>(mxm, m1, m3, xsf, w1sf, w3sf, offsets, G, d, f, rows_cap, hq, hsf, nullptr, s);
  if (e != cudaSuccess) return e;
  return mx::launch_mx<1>(mh, m2, m2, hsf, w2sf, w2sf, offsets, G, f, d, rows_cap, nullptr, nullptr, y, s);
}

}  // namespace moe
