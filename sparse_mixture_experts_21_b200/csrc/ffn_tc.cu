// Grouped SwiGLU expert FFN on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The Practice page's "专家并行与 all-to-all" points out that expert-contiguous rows
// let one grouped GEMM compute every expert at once instead of N small GEMMs; the
// expert itself is E(x) = W2 (silu(W1 x) * (W3 x)) (three matrices per expert, as
// in its "推理侧的路由稳定性" parameter count E x 3D^2).
//
// Two persistent launches over a tile list built on the device from `offsets`:
//   pass 0 (gate/up): H[r, n0:n0+128] = silu(X W1[g]^T) * (X W3[g]^T); the B tile
//          stacks 128 rows of W1 over 128 rows of W3, so one N = 256 MMA gives gate
//          and up for 128 hidden units and SwiGLU runs in the epilogue from TMEM.
//   pass 1 (down):    Y[r, n0:n0+256] = H W2[g]^T.
// Every MMA is tcgen05.mma.cta_group::1.kind::f16, M 128, N 256, K 16, bf16 in,
// fp32 accumulate in TMEM; operands come by TMA (128-byte swizzle, no multicast).
//
// Two tile shapes, one per pass:
//  * PAIR (pass 0, long K = d): a CTA tile is 256 rows of one group as two M = 128
//    sub-tiles sharing each B stage: per 64-wide K step it loads A0 16 KB + A1 16 KB
//    + B 32 KB and issues 2 x 4 MMAs, 64 bytes of operand traffic per MMA cycle
//    (96 with one 128-row tile), 3-stage ring.  A group's last tile with at most
//    128 rows loads and computes sub-tile 0 only, so padding stays at 128 rows.
//    TMEM holds both accumulators (2 x 256 columns); to hide the epilogue, the 8
//    epilogue warps drain accumulator 0 first, and as soon as it is free the MMA
//    warp computes sub-tile 0 of the next tile over the first resident K stages,
//    then waits for accumulator 1 and catches up sub-tile 1 on the same stages.
//  * SINGLE (pass 1, short K = f): 128-row tiles, 4-stage ring of 48 KB, two TMEM
//    accumulators used alternately so one tile's epilogue (4 warps) overlaps the
//    next tile's MMAs completely — with K = 2048 a tile is too short to absorb the
//    paired shape's epilogue bubble.
//
// Warp roles: 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2.. = epilogue
// (TMEM lane quarter = warp % 4).  Tiles are ordered group, n-tile, m-tile, so
// CTAs running together share weight tiles through L2.  Rows past a group's end
// are computed from whatever follows and never stored.  Every mbarrier wait is
// bounded; on timeout the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace tc {

constexpr int SUB = 128;                      // rows per MMA
constexpr int BK = 64;
constexpr int A_BYTES = SUB * BK * 2;         // 16 KB per 128-row A tile
constexpr int B_BYTES = 256 * BK * 2;         // 32 KB
constexpr int TMEM_COLS = 512;                // two 256-column fp32 accumulators
constexpr int kMaxGroups = 512;

template <bool PAIR>
struct Shape {
  static constexpr int BM = PAIR ? 2 * SUB : SUB;
  static constexpr int STAGES = PAIR ? 3 : 4;
  static constexpr int STAGE_BYTES = (PAIR ? 2 : 1) * A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = PAIR ? 8 : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
};

template <int STAGES>
struct __align__(8) TcShared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  int32_t goff[kMaxGroups + 1];   // group row offsets
  int32_t tpre[kMaxGroups + 1];   // prefix of full tiles (BM rows, or two sub-tiles) per group
  int32_t spre[kMaxGroups + 1];   // paired shape: prefix of tail tiles of at most 128 rows
};

template <bool PAIR>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Shape<PAIR>::STAGES * Shape<PAIR>::STAGE_BYTES +
         sizeof(TcShared<Shape<PAIR>::STAGES>);
}

template <class SH>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, SH* sh) {
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
  bool two;        // (paired shape) sub-tile 1 has rows
};

// Tile list.  Single shape: (group, n-tile, m-tile) over 128-row tiles.  Paired
// shape, in two phases so that tiles running side by side take the same time
// (CTAs that share a weight tile through L2 must stay in step, and a weight tile
// stays in L2 only for microseconds): first every tile with two sub-tiles
// (group, n-tile, m-tile), then every tail of at most 128 rows (group, n-tile).
template <bool PAIR, class SH>
__device__ __forceinline__ int find_group(const int32_t* pre, int G, int tiles_n, int L) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with pre[g] * tiles_n <= L
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <bool PAIR, class SH>
__device__ __forceinline__ Tile decode_tile(int L, const SH* sh, int G, int tiles_n, int BN) {
  constexpr int BM = PAIR ? 2 * SUB : SUB;
  Tile t;
  const int na = sh->tpre[G] * tiles_n;
  if (L < na) {
    const int g = find_group<PAIR, SH>(sh->tpre, G, tiles_n, L);
    const int local = L - sh->tpre[g] * tiles_n;
    const int mt = sh->tpre[g + 1] - sh->tpre[g];
    const int n_tile = local / mt, m_tile = local - n_tile * mt;
    t.g = g;
    t.row0 = sh->goff[g] + m_tile * BM;
    t.rows = min(BM, sh->goff[g + 1] - t.row0);
    t.n0 = n_tile * BN;
  } else {
    const int Lb = L - na;
    const int g = find_group<PAIR, SH>(sh->spre, G, tiles_n, Lb);
    const int rows_g = sh->goff[g + 1] - sh->goff[g];
    t.g = g;
    t.rows = rows_g % BM;
    t.row0 = sh->goff[g + 1] - t.rows;
    t.n0 = (Lb - sh->spre[g] * tiles_n) * BN;
  }
  t.two = t.rows > SUB;
  return t;
}

// Per-group tile prefixes, one warp.
template <bool PAIR, class SH>
__device__ void build_tile_table(SH* sh, const int32_t* offsets, int G, int lane) {
  constexpr int BM = PAIR ? 2 * SUB : SUB;
  int carry = 0, carry_s = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int mt = 0, st = 0;
    if (g < G) {
      const int o0 = offsets[g], o1 = offsets[g + 1];
      sh->goff[g] = o0;
      const int rows = o1 > o0 ? o1 - o0 : 0;
      if (PAIR) {
        const int rem = rows % BM;
        mt = rows / BM + (rem > SUB ? 1 : 0);
        st = (rem > 0 && rem <= SUB) ? 1 : 0;
      } else {
        mt = (rows + BM - 1) / BM;
      }
    }
    int incl = mt, incl_s = st;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      const int u = __shfl_up_sync(0xffffffffu, incl_s, o);
      if (lane >= o) { incl += v; incl_s += u; }
    }
    if (g < G) { sh->tpre[g + 1] = carry + incl; sh->spre[g + 1] = carry_s + incl_s; }
    carry += __shfl_sync(0xffffffffu, incl, 31);
    carry_s += __shfl_sync(0xffffffffu, incl_s, 31);
  }
  if (lane == 0) {
    sh->tpre[0] = 0;
    sh->spre[0] = 0;
    sh->goff[G] = offsets[G];
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Epilogue of one accumulator: TMEM columns [c_begin, c_end) of this warp's 32
// lanes -> bf16 rows of `out`.  MODE 0 pairs gate column c with up column 128 + c.
template <int MODE>
__device__ __forceinline__ void drain(uint32_t tbase, int c_begin, int c_end, bool row_ok,
                                      __nv_bfloat16* orow, int col0, int n_out) {
#pragma unroll 1
  for (int c = c_begin; c < c_end; c += 16) {
    float o[16];
    if (MODE == 0) {
      uint32_t gv[16], uv[16];
      tmem_ld16(tbase + c, gv);
      tmem_ld16(tbase + 128 + c, uv);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = silu_f(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
    } else {
      uint32_t v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = __uint_as_float(v[i]);
    }
    if (row_ok) {
      const int col = col0 + c;
      if (col + 8 <= n_out) stg16(orow + c, pack16(o, __nv_bfloat16()));
      if (col + 16 <= n_out) stg16(orow + c + 8, pack16(o + 8, __nv_bfloat16()));
    }
  }
}

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(Shape<PAIR>::THREADS, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const int32_t* __restrict__ offsets,
              int G, int K, int n_out, int64_t rows_cap, __nv_bfloat16* __restrict__ out) {
  using S = Shape<PAIR>;
  using SH = TcShared<S::STAGES>;
  constexpr int STAGES = S::STAGES, STAGE_BYTES = S::STAGE_BYTES;
  constexpr int BN = MODE == 0 ? 128 : 256;    // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  SH* sh = reinterpret_cast<SH*>(smem + (size_t)STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&sh->tfull[a], 1); mbar_init(&sh->tempty[a], S::EPI_WARPS); }
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
  if (warp == 2) build_tile_table<PAIR>(sh, offsets, G, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh->tmem_base;
  const int total = (sh->tpre[G] + (PAIR ? sh->spre[G] : 0)) * tiles_n;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile t = decode_tile<PAIR>(L, sh, G, tiles_n, BN);
        const bool two = PAIR && t.two;
        const int brow = t.g * n_out + t.n0;
        const uint32_t bytes = two ? STAGE_BYTES : A_BYTES + B_BYTES;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_or_abort(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* b = a + (PAIR ? 2 : 1) * A_BYTES;
          mbar_arrive_expect_tx(&sh->full[stage], bytes);
          tma_load_2d(&tmA, a, &sh->full[stage], kb * BK, t.row0);
          if (two) tma_load_2d(&tmA, a + A_BYTES, &sh->full[stage], kb * BK, t.row0 + SUB);
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
      constexpr uint32_t idesc = umma_idesc_bf16(SUB, 256);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      // MMAs of one K stage into accumulator `acc` from A sub-tile `sub`
      auto issue = [&](uint32_t st, int sub, uint32_t acc, bool first_kb) {
        const uint32_t base = smem_u32(smem + (size_t)st * STAGE_BYTES);
        const uint32_t a_addr = base + sub * A_BYTES;
        const uint32_t b_addr = base + (PAIR ? 2 : 1) * A_BYTES;
        const uint32_t d_tmem = tmem_base + acc * 256u;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32),
                   idesc, (!first_kb || kk != 0) ? 1u : 0u);
      };
      if constexpr (PAIR) {
        uint32_t use0 = 0, use1 = 0;       // completed uses of each accumulator
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
          const Tile t = decode_tile<PAIR>(L, sh, G, tiles_n, BN);
          if (!wait_or_abort(&sh->tempty[0], (use0 & 1u) ^ 1u, sh)) { ok = false; break; }
          tc_fence_after();
          // sub-tile 0 over the first P stages while accumulator 1 may still drain
          const int P = nkb < STAGES ? nkb : STAGES;
          const uint32_t st0 = stage;
          for (int j = 0; j < P; ++j) {
            if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
            tc_fence_after();
            issue(stage, 0, 0, j == 0);
            if (!t.two) umma_commit(&sh->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          if (t.two) {
            if (!wait_or_abort(&sh->tempty[1], (use1 & 1u) ^ 1u, sh)) { ok = false; break; }
            tc_fence_after();
            uint32_t s2 = st0;
            for (int j = 0; j < P; ++j) {
              issue(s2, 1, 1, j == 0);
              umma_commit(&sh->empty[s2]);
              if (++s2 == STAGES) s2 = 0;
            }
          }
          for (int kb = P; kb < nkb; ++kb) {
            if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
            tc_fence_after();
            issue(stage, 0, 0, false);
            if (t.two) issue(stage, 1, 1, false);
            umma_commit(&sh->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          umma_commit(&sh->tfull[0]);
          ++use0;
          if (t.two) {
            umma_commit(&sh->tfull[1]);
            ++use1;
          }
        }
      } else {
        uint32_t acc = 0, acc_phase = 0;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
          if (!wait_or_abort(&sh->tempty[acc], acc_phase ^ 1u, sh)) { ok = false; break; }
          tc_fence_after();
          for (int kb = 0; kb < nkb; ++kb) {
            if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
            tc_fence_after();
            issue(stage, 0, acc, kb == 0);
            umma_commit(&sh->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          umma_commit(&sh->tfull[acc]);
          acc ^= 1u;
          if (acc == 0) acc_phase ^= 1u;
        }
      }
      // every MMA of this CTA has finished once this barrier flips
      umma_commit(&sh->mma_done);
      mbar_wait(&sh->mma_done, 0);
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> global
    const int q = warp & 3;                   // TMEM lane quarter of this warp
    if constexpr (PAIR) {
      // Each warp copies its 32 lanes x 128 columns of an accumulator into registers
      // behind one wait, releases the accumulator, and only then converts and stores,
      // so the MMA warp waits for the TMEM copy, not for the global stores.
      const int half = (warp - 2) >> 2;       // column half handled by this warp
      uint32_t use0 = 0, use1 = 0;
      for (int L = blockIdx.x; L < total; L += gridDim.x) {
        const Tile t = decode_tile<PAIR>(L, sh, G, tiles_n, BN);
        bool ok = true;
        for (int sub = 0; sub < (t.two ? 2 : 1); ++sub) {
          uint32_t& use = sub == 0 ? use0 : use1;
          if (!wait_or_abort(&sh->tfull[sub], use & 1u, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + sub * 256u;
          uint32_t v[128];
          if (MODE == 0) {             // gate columns [64 h, 64 h + 64) and the matching up columns
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_ld16(tbase + half * 64 + 16 * j, v + 16 * j);
              tmem_ld16(tbase + 128 + half * 64 + 16 * j, v + 64 + 16 * j);
            }
          } else {                     // output columns [128 h, 128 h + 128)
#pragma unroll
            for (int j = 0; j < 8; ++j) tmem_ld16(tbase + half * 128 + 16 * j, v + 16 * j);
          }
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->tempty[sub]);
          ++use;
          const int r = sub * SUB + q * 32 + lane;
          const int64_t grow = (int64_t)t.row0 + r;
          if (r < t.rows && grow < rows_cap) {
            __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0;
            constexpr int NC = MODE == 0 ? 64 : 128;     // output columns of this thread
            const int c0 = half * NC;
#pragma unroll
            for (int j = 0; j < NC; j += 8) {
              float o[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = MODE == 0 ? silu_f(__uint_as_float(v[j + i])) * __uint_as_float(v[64 + j + i])
                                 : __uint_as_float(v[j + i]);
              if (t.n0 + c0 + j + 8 <= n_out) {
                uint4 pk;
                pk.x = pack_bf16x2(o[0], o[1]); pk.y = pack_bf16x2(o[2], o[3]);
                pk.z = pack_bf16x2(o[4], o[5]); pk.w = pack_bf16x2(o[6], o[7]);
                stg16(orow + c0 + j, pk);
              }
            }
          }
        }
        if (!ok) break;
      }
    } else {
      constexpr int CW = MODE == 0 ? 128 : 256;
      uint32_t acc = 0, acc_phase = 0;
      for (int L = blockIdx.x; L < total; L += gridDim.x) {
        const Tile t = decode_tile<PAIR>(L, sh, G, tiles_n, BN);
        if (!wait_or_abort(&sh->tfull[acc], acc_phase, sh)) break;
        tc_fence_after();
        const int r = q * 32 + lane;
        const int64_t grow = (int64_t)t.row0 + r;
        drain<MODE>(tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256u, 0, CW,
                    r < t.rows && grow < rows_cap, out + grow * (int64_t)n_out + t.n0, t.n0, n_out);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tempty[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int MODE, bool PAIR>
cudaError_t launch_pass(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const int32_t* offsets, int G, int K, int n_out, int64_t rows_cap,
                        void* out, cudaStream_t s) {
  constexpr int BN = MODE == 0 ? 128 : 256;
  constexpr size_t SMEM = smem_bytes<PAIR>();
  const cudaError_t e = ensure_smem_attr((const void*)ffn_tc_kernel<MODE, PAIR>, (int)SMEM);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + Shape<PAIR>::BM - 1) / Shape<PAIR>::BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  ffn_tc_kernel<MODE, PAIR><<<grid, Shape<PAIR>::THREADS, SMEM, s>>>(
      a, b0, b1, offsets, G, K, n_out, rows_cap, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_ffn_bf16(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                            const void* w1, const void* w3, const void* w2, int d, int f, void* h,
                            void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > tc::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mx, m1, m3, mh, m2;
  if (!make_map_bf16(&mx, x_rows, rows_cap, d, tc::SUB) || !make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) ||
      !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128) || !make_map_bf16(&mh, h, rows_cap, f, tc::SUB) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = tc::launch_pass<0, true>(mx, m1, m3, offsets, G, d, f, rows_cap, h, s);
  if (e != cudaSuccess) return e;
  return tc::launch_pass<1, false>(mh, m2, m2, offsets, G, f, d, rows_cap, y, s);
}

}  // namespace moe
