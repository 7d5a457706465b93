// Down projection of the grouped SwiGLU expert FFN: Y[r, n0:n0+256] = H W2[g]^T over
// every group's rows, tcgen05 tensor cores (see ffn_tc.cu for the gate/up pass and
// the source passages).
//
// 128-row tiles of one group in (group, n-tile, m-tile) order; persistent CTAs take
// tiles round-robin (every tile has the same length, so CTAs that share a weight
// tile through L2 stay in step).  4-stage ring of 48 KB (A 16 KB + W2 tile 32 KB per
// 64-wide K step); two 256-column TMEM accumulators used alternately, so one tile's
// epilogue (4 warps) overlaps the next tile's MMAs completely -- with K = d_ff a tile
// is too short to absorb an epilogue bubble.  A group's last tile computes on
// whatever rows follow and stores only the group's own.  Warp roles: 0 = TMA
// producer, 1 = TMEM allocator + MMA issuer, 2..5 = epilogue.  Every wait is bounded;
// on timeout the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its own copies and
// MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace dn {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGES = 4;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int kMaxGroups = 512;

struct __align__(8) DnShared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  int32_t goff[kMaxGroups + 1];
  int32_t tpre[kMaxGroups + 1];   // prefix of 128-row tiles per group
};

constexpr size_t kSmem = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(DnShared);

__device__ __forceinline__ bool wait_dn(uint64_t* bar, uint32_t parity, DnShared* sh) {
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

struct DTile {
  int g, row0, rows, n0;
};

__device__ __forceinline__ DTile decode(int L, const DnShared* sh, int G, int tiles_n) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with tpre[g] * tiles_n <= L
    const int mid = (lo + hi + 1) >> 1;
    if (sh->tpre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int local = L - sh->tpre[g] * tiles_n;
  const int mt = sh->tpre[g + 1] - sh->tpre[g];
  const int n_tile = local / mt, m_tile = local - n_tile * mt;
  DTile t;
  t.g = g;
  t.row0 = sh->goff[g] + m_tile * BM;
  t.rows = min(BM, sh->goff[g + 1] - t.row0);
  t.n0 = n_tile * BN;
  return t;
}

__global__ void __launch_bounds__(THREADS, 1)
ffn_down_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const int32_t* __restrict__ offsets, int G, int K, int n_out, int64_t rows_cap,
                __nv_bfloat16* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  DnShared* sh = reinterpret_cast<DnShared*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&sh->tfull[a], 1); mbar_init(&sh->tempty[a], EPI_WARPS); }
    mbar_init(&sh->mma_done, 1);
    sh->abort = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
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
    // ---------------- TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const DTile t = decode(L, sh, G, tiles_n);
        const int brow = t.g * n_out + t.n0;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_dn(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES);
          tma_load_2d(&tmA, a, &sh->full[stage], kb * BK, t.row0);
          tma_load_2d(&tmB, a + A_BYTES, &sh->full[stage], kb * BK, brow);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // drain this CTA's own copies still in flight before leaving
        for (int i = 1; i <= min(issued, STAGES); ++i) {
          const int st = ((int)stage - i + 2 * STAGES) % STAGES;
          mbar_wait(&sh->full[st], ((int)stage - i < 0) ? (phase ^ 1u) : phase);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        if (!wait_dn(&sh->tempty[acc], acc_phase ^ 1u, sh)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256u;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_dn(&sh->full[stage], phase, sh)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                     (kb != 0 || kk != 0) ? 1u : 0u);
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
    // ---------------- epilogue: TMEM -> registers -> bf16 rows
    const int q = warp & 3;
    uint32_t acc = 0, acc_phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const DTile t = decode(L, sh, G, tiles_n);
      if (!__all_sync(0xffffffffu, wait_dn(&sh->tfull[acc], acc_phase, sh))) break;
      tc_fence_after();
      const int r = q * 32 + lane;
      const int64_t grow = (int64_t)t.row0 + r;
      const bool row_ok = r < t.rows && grow < rows_cap;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256u;
      __nv_bfloat16* orow = out + grow * (int64_t)n_out + t.n0;
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tmem_ld16(tb + c, v);
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
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dn

// H [rows_cap, f] (tensor map `mh`, 128-row boxes) times W2 [G d, f] (`m2`, 256-row
// boxes) -> Y [rows_cap, d].
cudaError_t launch_ffn_down(const CUtensorMap& mh, const CUtensorMap& m2, const int32_t* offsets, int G, int f,
                            int d, int64_t rows_cap, void* y, cudaStream_t s) {
  const cudaError_t e = ensure_smem_attr((const void*)dn::ffn_down_kernel, (int)dn::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (d + dn::BN - 1) / dn::BN;
  const int64_t max_tiles = ((rows_cap + dn::BM - 1) / dn::BM + G) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  dn::ffn_down_kernel<<<grid, dn::THREADS, dn::kSmem, s>>>(mh, m2, offsets, G, f, d, rows_cap,
                                                           static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

}  // namespace moe
