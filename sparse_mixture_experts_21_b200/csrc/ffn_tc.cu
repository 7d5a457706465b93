// Grouped SwiGLU expert FFN on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The Practice page's "专家并行与 all-to-all" points out that expert-contiguous rows
// let one grouped GEMM compute every expert at once instead of N small GEMMs; the
// expert itself is E(x) = W2 (silu(W1 x) * (W3 x)) (three matrices per expert, as
// in its "推理侧的路由稳定性" parameter count E x 3D^2).
//
// Two persistent launches over a tile list built on the device from `offsets`:
//   pass 0 (gate/up): H[r, n0:n0+128] = silu(X W1[g]^T) * (X W3[g]^T); each MMA
//          has N = 256 = 128 gate columns followed by 128 up columns, so SwiGLU is
//          applied in the epilogue straight from TMEM.
//   pass 1 (down):    Y[r, n0:n0+256] = H W2[g]^T.
// Tile 128 rows x 256 MMA columns, K step 64 (one 128-byte swizzle atom), 4-stage
// TMA ring, two TMEM accumulators (2 x 256 fp32 columns) so the epilogue of one
// tile overlaps the MMAs of the next.  Warp roles: 0 = TMA producer, 1 = TMEM
// allocator + MMA issuer, 2..5 = epilogue (TMEM lane quarter = warp % 4).
// Tiles are ordered group-major, then n-tile, then m-tile, so CTAs running at the
// same time share the same weight tile through L2.  Rows of a partial m-tile past
// the group end are computed from whatever rows follow and never stored.
// Every mbarrier wait is bounded; on timeout the kernel records
// MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = 256 * BK * 2;         // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int kThreads = 192;
constexpr int kMaxGroups = 512;

struct __align__(8) TcShared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  int32_t goff[kMaxGroups + 1];   // group row offsets
  int32_t tpre[kMaxGroups + 1];   // prefix of m-tiles per group
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(TcShared);

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, TcShared* sh) {
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
  int g, row0, rows, n0;
};

__device__ __forceinline__ Tile decode_tile(int L, const TcShared* sh, int G, int tiles_n, int BN) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with tpre[g] * tiles_n <= L
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
  return t;
}

// Per-group m-tile prefix, one warp.
__device__ void build_tile_table(TcShared* sh, const int32_t* offsets, int G, int lane) {
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
  if (lane == 0) {
    sh->tpre[0] = 0;
    sh->goff[G] = offsets[G];
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const int32_t* __restrict__ offsets,
              int G, int K, int n_out, int64_t rows_cap, __nv_bfloat16* __restrict__ out) {
  constexpr int BN = MODE == 0 ? 128 : 256;    // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  TcShared* sh = reinterpret_cast<TcShared*>(smem + (size_t)STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&sh->tfull[a], 1); mbar_init(&sh->tempty[a], 4); }
    mbar_init(&sh->mma_done, 1);
    sh->abort = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    if (MODE == 0) prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) build_tile_table(sh, offsets, G, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh->tmem_base;
  const int total = sh->tpre[G] * tiles_n;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile t = decode_tile(L, sh, G, tiles_n, BN);
        const int brow = t.g * n_out + t.n0;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_or_abort(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
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
        // drain this CTA's own copies still in flight before leaving
        for (int i = 1; i <= min(issued, STAGES); ++i) {
          const int s = ((int)stage - i + 2 * STAGES) % STAGES;
          const uint32_t ph = ((int)stage - i < 0) ? (phase ^ 1u) : phase;
          mbar_wait(&sh->full[s], ph);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, 256);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        if (!wait_or_abort(&sh->tempty[acc], acc_phase ^ 1u, sh)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256u;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32),
                     idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&sh->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&sh->tfull[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every MMA of this CTA has finished once this barrier flips
      umma_commit(&sh->mma_done);
      mbar_wait(&sh->mma_done, 0);
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> global
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const Tile t = decode_tile(L, sh, G, tiles_n, BN);
      if (!wait_or_abort(&sh->tfull[acc], acc_phase, sh)) break;
      tc_fence_after();
      const int64_t grow = (int64_t)t.row0 + r;
      const bool row_ok = r < t.rows && grow < rows_cap;
      __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256u;
      if (MODE == 0) {
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          uint32_t gv[16], uv[16];
          tmem_ld16(tbase + c, gv);
          tmem_ld16(tbase + 128 + c, uv);
          tmem_ld_wait();
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = silu_f(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
          if (row_ok) {
            const int col = t.n0 + c;
            if (col + 8 <= n_out) stg16(orow + c, pack16(h, __nv_bfloat16()));
            if (col + 16 <= n_out) stg16(orow + c + 8, pack16(h + 8, __nv_bfloat16()));
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 256; c += 16) {
          uint32_t v[16];
          tmem_ld16(tbase + c, v);
          tmem_ld_wait();
          float o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __uint_as_float(v[i]);
          if (row_ok) {
            const int col = t.n0 + c;
            if (col + 8 <= n_out) stg16(orow + c, pack16(o, __nv_bfloat16()));
            if (col + 16 <= n_out) stg16(orow + c + 8, pack16(o + 8, __nv_bfloat16()));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->tempty[acc]);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int MODE>
cudaError_t launch_pass(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const int32_t* offsets, int G, int K, int n_out, int64_t rows_cap,
                        void* out, cudaStream_t s) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ffn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + BM - 1) / BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  ffn_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(a, b0, b1, offsets, G, K, n_out, rows_cap,
                                                          static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace tc


cudaError_t launch_ffn_bf16(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                            const void* w1, const void* w3, const void* w2, int d, int f, void* h,
                            void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > tc::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mx, m1, m3, mh, m2;
  if (!make_map_bf16(&mx, x_rows, rows_cap, d, tc::BM) || !make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) ||
      !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128) || !make_map_bf16(&mh, h, rows_cap, f, tc::BM) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = tc::launch_pass<0>(mx, m1, m3, offsets, G, d, f, rows_cap, h, s);
  if (e != cudaSuccess) return e;
  return tc::launch_pass<1>(mh, m2, m2, offsets, G, f, d, rows_cap, y, s);
}

}  // namespace moe
