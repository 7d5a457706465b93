// Grouped SwiGLU expert FFN on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The Practice page's "专家并行与 all-to-all" points out that expert-contiguous rows
// let one grouped GEMM compute every expert at once instead of N small GEMMs; the
// expert itself is E(x) = W2 (silu(W1 x) * (W3 x)) (three matrices per expert, as
// in its "推理侧的路由稳定性" parameter count E x 3D^2).
//
// Two persistent launches of one kernel over tile lists built on the device from
// `offsets`:
//   gate/up (MODE 0): H[r, n0:n0+128] = silu(X W1[g]^T) * (X W3[g]^T); the weight
//          tile stacks 128 rows of W1 over 128 rows of W3, so one N = 256 MMA gives
//          gate and up for 128 hidden units and SwiGLU runs in the epilogue from TMEM.
//   down (MODE 1):    Y[r, n0:n0+256] = H W2[g]^T.
// Every MMA is tcgen05.mma.cta_group::1.kind::f16 (bf16 in, fp32 accumulate in
// TMEM); operands come by TMA (128-byte swizzle, no multicast).
//
// A CTA tile is up to two 128-row sub-tiles of one group sharing each weight stage.
// Per 64-wide K step a stage holds A0 16 KB + A1 16 KB + W 32 KB (the weight tile),
// 64 bytes of operand traffic per MMA cycle for two full sub-tiles (96 with one
// 128-row tile); 3-stage ring; TMEM holds two 256-column fp32 accumulators, one per
// sub-tile.  To hide the epilogue, the 8 epilogue warps drain accumulator 0 first,
// and as soon as it is free the MMA warp computes sub-tile 0 of the next tile over
// the first resident stages, then waits for accumulator 1 and catches up sub-tile 1
// on the same stages.
//
// No padding rows.  A group of R rows is cut into floor(R / 128) full 128-row
// sub-tiles (paired two by two) and a ragged tail of r = R mod 128 rows.  The tail
// is computed transposed ("swapped"): the weight tile already in shared memory is
// the MMA's A operand (M = 128 weight rows, i.e. output columns) and the r tail rows
// are its B operand (N = r rounded up to 16), so the tail costs its own MMA work,
// not that of a 128-row tile, and reuses the weight stages of the group's last full
// sub-tile.  Kinds of tile:
//   PAIR   two full sub-tiles;
//   SINGLE one full sub-tile (an odd count of full sub-tiles), no tail;
//   ST     one full sub-tile + the group's tail as sub-tile 1 (swapped);
//   T      the tail alone (an even count of full sub-tiles, or R < 128).
// The swapped sub-tile writes D^T into accumulator 1: weight rows 0..127 into
// columns [0, n) and rows 128..255 into columns [128, 128 + n) (gate/up: W1 and W3,
// so gate and up of one hidden unit share a TMEM lane; down: the two 128-column
// halves of the output tile).
//
// Tile order and scheduling: group, n-tile, then that (group, n-tile)'s PAIR tiles
// followed by its extra tile.  Tiles are claimed dynamically -- the producer warp
// takes the next index from a per-launch global counter and hands it to the MMA
// and epilogue warps through a small shared-memory queue -- so the tiles in flight
// are always a contiguous window of the list and the CTAs that share a weight tile
// run together, whatever the tiles' lengths (a static round-robin assignment lets
// CTAs drift apart and stream weight tiles from DRAM again).  The last CTA to
// finish resets the counter.
//
// Warp roles: 0 = TMA producer (and tile claims), 1 = TMEM allocator + MMA issuer,
// 2.. = epilogue (TMEM lane quarter = warp % 4).  Every mbarrier wait is bounded; on
// timeout the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs,
// frees TMEM and returns.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace tc {

constexpr int SUB = 128;                      // rows per MMA (full sub-tile)
constexpr int BK = 64;
constexpr int A_BYTES = SUB * BK * 2;         // 16 KB per 128-row A tile
constexpr int W_BYTES = 256 * BK * 2;         // 32 KB weight tile
constexpr int STAGES = 3;
constexpr int STAGE_BYTES = 2 * A_BYTES + W_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int TMEM_COLS = 512;                // two 256-column fp32 accumulators
constexpr int TAIL_BOX = 16;                  // rows per TMA box of a tail (swapped) operand
constexpr int kMaxGroups = 512;

enum TileKind { K_PAIR = 0, K_SINGLE = 1, K_ST = 2, K_T = 3 };

constexpr int TQ = 4;                         // tile indices in flight from the producer
constexpr int kCtrSlots = 64;                 // per-launch tile counters (rotating)

struct __align__(8) TcShared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t tq_full[TQ];
  uint64_t tq_empty[TQ];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile int32_t abort;
  volatile int32_t tq[TQ];        // claimed tile indices (>= total: no more tiles)
  int32_t goff[kMaxGroups + 3];   // group row offsets (then an empty gap and the extra group)
  int32_t tpre[kMaxGroups + 3];   // prefix over groups of (PAIR tiles + extra tile) per n-tile
};

// Per-launch tile counters: [slot][0] = next tile to claim, [slot][1] = CTAs done.
// Each launch takes the next slot; its last CTA puts both back to 0.  Launches more
// than kCtrSlots apart may share a slot (the earlier one has long finished).
__device__ int32_t g_tile_ctr[kCtrSlots][2];

// Both passes stage their output through shared memory for TMA stores: one 32-row x
// 32-column bf16 box (2 KB, 64-byte swizzle) per epilogue warp.
constexpr int OUT_BOX = 2048;
constexpr size_t kSharedPad = (sizeof(TcShared) + 1023) / 1024 * 1024;
constexpr size_t kSmem = 1024 + (size_t)STAGES * STAGE_BYTES + kSharedPad + (size_t)EPI_WARPS * OUT_BOX;
static_assert(kSmem <= 232448, "shared memory per CTA");

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
  int g, n0, kind;
  int row0;          // first row of the full sub-tile(s)
  int trow0, tr;     // tail: first row and row count (kinds ST, T)
  int tn;            // tail rows rounded up to TAIL_BOX (the swapped MMA's N)
  __device__ bool has0() const { return kind != K_T; }
  __device__ bool has1() const { return kind != K_SINGLE; }
  __device__ bool swap1() const { return kind >= K_ST; }
};

__device__ __forceinline__ int find_group(const int32_t* pre, int G, int tiles_n, int L) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with pre[g] * tiles_n <= L
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] * tiles_n <= L) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ Tile decode_tile(int L, const TcShared* sh, int G, int tiles_n, int BN) {
  Tile t;
  const int g = find_group(sh->tpre, G, tiles_n, L);
  const int per = sh->tpre[g + 1] - sh->tpre[g];          // tiles of group g per n-tile
  const int local = L - sh->tpre[g] * tiles_n;
  const int n_tile = local / per, j = local - n_tile * per;
  const int rows = sh->goff[g + 1] - sh->goff[g];
  const int full = rows / SUB, r = rows - full * SUB;
  t.g = g;
  t.n0 = n_tile * BN;
  if (j < full / 2) {
    t.kind = K_PAIR;
    t.row0 = sh->goff[g] + j * 2 * SUB;
    t.trow0 = 0;
    t.tr = 0;
    t.tn = 0;
  } else {
    t.kind = (full & 1) ? (r > 0 ? K_ST : K_SINGLE) : K_T;
    t.row0 = sh->goff[g] + (full & ~1) * SUB;
    t.trow0 = sh->goff[g + 1] - r;
    t.tr = r;
    t.tn = (r + TAIL_BOX - 1) / TAIL_BOX * TAIL_BOX;
  }
  return t;
}

// Tiles of a group of `rows` rows per n-tile: its PAIR tiles + at most one more.
__device__ __forceinline__ int group_tiles(int rows) {
  const int full = rows / SUB;
  return full / 2 + (((full & 1) || rows % SUB) ? 1 : 0);
}

// Per-group tile prefixes, one warp.  With a dense extra group (rows_x > 0) the
// list goes on with an empty group over rows [offsets[G], rows_cap) and the extra
// group G + 1 over rows [rows_cap, rows_cap + rows_x): its rows are numbered as its
// output rows.
__device__ void build_tile_table(TcShared* sh, const int32_t* offsets, int G, int rows_x, int rows_cap,
                                 int lane) {
  int carry = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int mt = 0;
    if (g < G) {
      const int o0 = offsets[g], o1 = offsets[g + 1];
      sh->goff[g] = o0;
      mt = group_tiles(o1 > o0 ? o1 - o0 : 0);
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
    if (rows_x > 0) {
      sh->goff[G + 1] = rows_cap;
      sh->goff[G + 2] = rows_cap + rows_x;
      sh->tpre[G + 1] = carry;
      sh->tpre[G + 2] = carry + group_tiles(rows_x);
    }
  }
}

// Consumer side of the tile queue: the i-th claimed tile index (>= total: done).
__device__ __forceinline__ bool next_tile(TcShared* sh, uint32_t i, int* L) {
  const uint32_t slot = i % TQ, ph = (i / TQ) & 1u;
  if (!wait_or_abort(&sh->tq_full[slot], ph, sh)) return false;
  *L = sh->tq[slot];
  return true;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Swapped (tail) epilogue.  The epilogue loads the same TMEM columns for a normal
// and for a swapped sub-tile (gate/up: columns [64 h, 64 h + 64) and 128 + those;
// down: [128 h, 128 h + 128)); only their meaning differs.  Normal: the lane is a
// row and the columns are output columns.  Swapped: the lane is an output column
// and the columns are tail rows -- gate/up: warp half h holds tail rows
// [64 h, 64 h + 64) of hidden unit n0 + 32 q + lane (gate at v[i], up at v[64 + i]);
// down: warp half h holds every tail row of output column n0 + 128 h + 32 q + lane.
// Columns past the tail hold stale values and are never stored.
template <int MODE>
__device__ __forceinline__ void store_swapped(const uint32_t* v, const Tile& t, int half, int q, int lane,
                                              int n_out, int64_t rows_cap, __nv_bfloat16* out) {
  const int col = t.n0 + (MODE == 0 ? 0 : 128 * half) + 32 * q + lane;
  const int64_t lim64 = rows_cap - t.trow0;
  const int lim = (int)(lim64 < t.tr ? lim64 : t.tr);        // tail rows to store
  if (col >= n_out) return;
  const int64_t ld = n_out;
  __nv_bfloat16* p = out + (int64_t)t.trow0 * ld + col;
  // one running pointer (a chain of adds), so the unrolled loop does not keep an
  // address per row live
  if (MODE == 0) {
    const int n = lim - half * 64;
    p += (int64_t)(half * 64) * ld;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if (i < n) *p = __float2bfloat16_rn(silu_f(__uint_as_float(v[i])) * __uint_as_float(v[64 + i]));
      asm volatile("" : "+l"(p));
      p += ld;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 128; ++i) {
      if (i < lim) *p = __float2bfloat16_rn(__uint_as_float(v[i]));
      asm volatile("" : "+l"(p));
      p += ld;
    }
  }
}

// Token of permuted row `row` for the gathering producer: an id outside [0, T) is
// recorded as MOE_ERR_INVALID_ARG and replaced by token 0.
__device__ __forceinline__ int32_t token_at(const int32_t* __restrict__ token_of_row, int64_t row, int T) {
  const int32_t v = token_of_row[row];
  if ((uint32_t)v >= (uint32_t)T) {
    flag_invalid_index();
    return 0;
  }
  return v;
}

// MODE 0: gate/up (B = W1 rows over W3 rows, maps tmB0 / tmB1, 128-row boxes; the
// epilogue applies SwiGLU); MODE 1: down (B = one 256-row W2 box, map tmB0).
// GATHER = false: A rows come from the expert-ordered rows (map tmA, 128-row boxes;
// tmAt, 16-row boxes for the tails).  GATHER = true (gate/up only): row r of group g
// is token token_of_row[r] of x [T, K] at xsrc, copied by the producer warp with
// cp.async (tmA, tmAt unused), so the expert-ordered copy of x is never written.
// The dense extra group (the shared expert run inside the same launches): its
// input rows are rows a_base .. a_base + rows - 1 of map a (128-row boxes; at: the
// tail boxes), its weights b0 / b1 (as for the groups); its outputs are rows
// rows_cap .. rows_cap + rows - 1 of the pass's output.  rows = 0: none.  In the
// tile list it is group G + 1, after an empty group G over the unused rows
// [offsets[G], rows_cap).
struct ExtraGroup {
  CUtensorMap a, at, b0, b1;
  int a_base;
  int rows;
};

template <int MODE, bool GATHER>
__global__ void __launch_bounds__(THREADS, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAt,
              const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
              const int32_t* __restrict__ offsets, int G, int K, int n_out, int64_t rows_cap,
              __nv_bfloat16* __restrict__ out, int ctr_slot, const int32_t* __restrict__ token_of_row,
              int T, const uint8_t* __restrict__ xsrc, const __grid_constant__ ExtraGroup xg,
              const __grid_constant__ CUtensorMap tmY) {
  static_assert(MODE == 0 || !GATHER, "only the gate/up pass gathers its rows");
  constexpr int BN = MODE == 0 ? 128 : 256;    // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  TcShared* sh = reinterpret_cast<TcShared*>(smem + (size_t)STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (n_out + BN - 1) / BN;
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    // a stage's full barrier: one arrival (with the TMA bytes), or, gathering, one per
    // lane of the producer warp
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], GATHER ? 32 : 1); mbar_init(&sh->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&sh->tfull[a], 1); mbar_init(&sh->tempty[a], EPI_WARPS); }
    for (int q = 0; q < TQ; ++q) { mbar_init(&sh->tq_full[q], 1); mbar_init(&sh->tq_empty[q], 1 + EPI_WARPS); }
    mbar_init(&sh->mma_done, 1);
    sh->abort = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmAt);
    prefetch_tmap(&tmB0);
    if (MODE == 0) prefetch_tmap(&tmB1);
    prefetch_tmap(&tmY);
    if (xg.rows > 0) {
      prefetch_tmap(&xg.a);
      prefetch_tmap(&xg.at);
      prefetch_tmap(&xg.b0);
      if (MODE == 0) prefetch_tmap(&xg.b1);
    }
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  const int rows_x = xg.rows;
  if (warp == 2) build_tile_table(sh, offsets, G, rows_x, (int)rows_cap, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh->tmem_base;
  const int Gt = G + (rows_x > 0 ? 2 : 0);     // groups in the tile list
  const int total = sh->tpre[Gt] * tiles_n;
  int32_t* ctr = g_tile_ctr[ctr_slot];

  if (warp == 0 && GATHER) {
    // ---------------- tile claims + gathering producer (whole warp)
    // A routed operand's rows are copied from x with cp.async: one instruction moves
    // 4 rows x 128 bytes (8 lanes per row, a 16-byte chunk each) into the 128-byte
    // swizzled layout of a TMA box, so 32 instructions fill a 128-row operand per K
    // step; token ids are read once per tile.  The weight tile, and the extra group's
    // rows, come by TMA.  A stage's barrier expects the TMA bytes and 32 arrivals, one
    // per lane, each made by the hardware once that lane's copies have landed; the MMA
    // warp fences them for the tensor cores' async-proxy reads after its wait.
    const int cl = lane & 7, rq = lane >> 3;    // 16-byte chunk of a row; row within a group of 4
    const size_t row_bytes = (size_t)K * 2;
    uint32_t stage = 0, phase = 0;
    int issued = 0;
    bool ok = true;
    // the lane's rows 4 j + rq of an operand, j < nj, copied into the box at `dst`
    auto gather = [&](uint32_t dst, const int32_t* ids, int nj, int kb) {
      const uint8_t* col = xsrc + (size_t)kb * (BK * 2) + cl * 16;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nj) {
          const int row = 4 * j + rq;
          cp_async16(dst + row * (BK * 2) + ((cl ^ (row & 7)) << 4), col + (size_t)ids[j] * row_bytes);
        }
      }
    };
    for (uint32_t i = 0; ok; ++i) {
      const uint32_t qs = i % TQ, qph = (i / TQ) & 1u;
      int L = -1;
      if (lane == 0 && wait_or_abort(&sh->tq_empty[qs], qph ^ 1u, sh)) {
        L = atomicAdd(&ctr[0], 1);
        sh->tq[qs] = L;
        mbar_arrive(&sh->tq_full[qs]);
      }
      L = __shfl_sync(0xffffffffu, L, 0);
      if (L < 0) { ok = false; break; }
      if (L >= total) break;
      Tile t = decode_tile(L, sh, Gt, tiles_n, BN);
      // the extra group reads its rows by TMA from its own maps, rows counted from its first row
      const bool ex = t.g == G + 1;
      const CUtensorMap* mB0 = ex ? &xg.b0 : &tmB0;
      const CUtensorMap* mB1 = ex ? &xg.b1 : &tmB1;
      if (ex) { t.row0 += xg.a_base - (int)rows_cap; t.trow0 += xg.a_base - (int)rows_cap; }
      const int brow = (ex ? 0 : t.g * n_out) + t.n0;
      const uint32_t tx = W_BYTES + (ex ? (t.has0() ? A_BYTES : 0) + (t.kind == K_PAIR ? A_BYTES : 0) +
                                              (t.swap1() ? t.tn * BK * 2 : 0)
                                         : 0);
      // token ids of this lane's rows; a row at or past `lim` (past the group's tail,
      // or past rows_cap) reads token 0 and feeds output that is never stored
      int32_t id0[32], id1[32];
      auto ids = [&](int64_t first, int64_t lim, int32_t* r) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int64_t row = first + 4 * j + rq;
          r[j] = row < lim ? token_at(token_of_row, row, T) : 0;
        }
      };
      const int nj1 = t.kind == K_PAIR ? 32 : (t.swap1() ? t.tn / 4 : 0);
      if (!ex) {
        if (t.has0()) ids(t.row0, rows_cap, id0);
        if (t.kind == K_PAIR) ids((int64_t)t.row0 + SUB, rows_cap, id1);
        else if (t.swap1()) ids(t.trow0, min((int64_t)t.trow0 + t.tr, rows_cap), id1);
      }
      for (int kb = 0; kb < nkb; ++kb) {
        const bool w = lane == 0 ? wait_or_abort(&sh->empty[stage], phase ^ 1u, sh) : true;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
        uint8_t* b = a + 2 * A_BYTES;
        if (lane == 0) {
          mbar_expect_tx(&sh->full[stage], tx);
          if (ex) {
            if (t.has0()) tma_load_2d(&xg.a, a, &sh->full[stage], kb * BK, t.row0);
            if (t.kind == K_PAIR) tma_load_2d(&xg.a, a + A_BYTES, &sh->full[stage], kb * BK, t.row0 + SUB);
            if (t.swap1())
              for (int j = 0; j < t.tn / TAIL_BOX; ++j)
                tma_load_2d(&xg.at, a + A_BYTES + j * TAIL_BOX * BK * 2, &sh->full[stage], kb * BK,
                            t.trow0 + j * TAIL_BOX);
          }
          tma_load_2d(mB0, b, &sh->full[stage], kb * BK, brow);
          if (MODE == 0) tma_load_2d(mB1, b + W_BYTES / 2, &sh->full[stage], kb * BK, brow);
        }
        __syncwarp();
        if (!ex) {
          if (t.has0()) gather(smem_u32(a), id0, 32, kb);
          if (nj1) gather(smem_u32(a + A_BYTES), id1, nj1, kb);
        }
        cp_async_arrive_noinc(&sh->full[stage]);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    // this lane's copies have landed; after an abort, this CTA's own TMA copies still
    // in flight are drained before leaving
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok && lane == 0) {
      for (int i = 1; i <= min(issued, STAGES); ++i) {
        const int s = ((int)stage - i + 2 * STAGES) % STAGES;
        const uint32_t ph = ((int)stage - i < 0) ? (phase ^ 1u) : phase;
        mbar_wait(&sh->full[s], ph);
      }
    }
  } else if (warp == 0) {
    // ---------------- tile claims + TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (uint32_t i = 0; ok; ++i) {
        // claim the next tile and hand its index to the MMA and epilogue warps
        const uint32_t qs = i % TQ, qph = (i / TQ) & 1u;
        if (!wait_or_abort(&sh->tq_empty[qs], qph ^ 1u, sh)) { ok = false; break; }
        const int L = atomicAdd(&ctr[0], 1);
        sh->tq[qs] = L;
        mbar_arrive(&sh->tq_full[qs]);
        if (L >= total) break;
        Tile t = decode_tile(L, sh, Gt, tiles_n, BN);
        // the extra group reads its own maps, rows counted from its first row
        const bool ex = t.g == G + 1;
        const CUtensorMap* mA = ex ? &xg.a : &tmA;
        const CUtensorMap* mAt = ex ? &xg.at : &tmAt;
        const CUtensorMap* mB0 = ex ? &xg.b0 : &tmB0;
        const CUtensorMap* mB1 = ex ? &xg.b1 : &tmB1;
        if (ex) { t.row0 += xg.a_base - (int)rows_cap; t.trow0 += xg.a_base - (int)rows_cap; }
        const int brow = (ex ? 0 : t.g * n_out) + t.n0;
        const uint32_t bytes = (t.has0() ? A_BYTES : 0) + (t.kind == K_PAIR ? A_BYTES : 0) +
                               (t.swap1() ? t.tn * BK * 2 : 0) + W_BYTES;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_or_abort(&sh->empty[stage], phase ^ 1u, sh)) { ok = false; break; }
          uint8_t* a = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* b = a + 2 * A_BYTES;
          mbar_arrive_expect_tx(&sh->full[stage], bytes);
          if (t.has0()) tma_load_2d(mA, a, &sh->full[stage], kb * BK, t.row0);
          if (t.kind == K_PAIR) tma_load_2d(mA, a + A_BYTES, &sh->full[stage], kb * BK, t.row0 + SUB);
          if (t.swap1())
            for (int j = 0; j < t.tn / TAIL_BOX; ++j)
              tma_load_2d(mAt, a + A_BYTES + j * TAIL_BOX * BK * 2, &sh->full[stage], kb * BK,
                          t.trow0 + j * TAIL_BOX);
          tma_load_2d(mB0, b, &sh->full[stage], kb * BK, brow);
          if (MODE == 0) tma_load_2d(mB1, b + W_BYTES / 2, &sh->full[stage], kb * BK, brow);
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
      // normal sub-tile: D[128 rows, 256] (+)= A_sub . W^T into accumulator `sub`
      auto issue = [&](uint32_t st, int sub, bool first_kb) {
        const uint32_t base = smem_u32(smem + (size_t)st * STAGE_BYTES);
        const uint32_t a_addr = base + sub * A_BYTES;
        const uint32_t b_addr = base + 2 * A_BYTES;
        const uint32_t d_tmem = tmem_base + sub * 256u;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32),
                   idesc, (!first_kb || kk != 0) ? 1u : 0u);
      };
      // swapped tail in sub-tile 1: D^T[128 weight rows, tn] (+)= W_half . Tail^T, the two
      // 128-row halves of the weight tile into columns [0, tn) and [128, 128 + tn) of
      // accumulator 1
      auto issue_swapped = [&](uint32_t st, int tn, bool first_kb) {
        const uint32_t base = smem_u32(smem + (size_t)st * STAGE_BYTES);
        const uint32_t tail_addr = base + A_BYTES;
        const uint32_t w_addr = base + 2 * A_BYTES;
        const uint32_t idesc_t = umma_idesc_bf16(SUB, tn);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t d_tmem = tmem_base + 256u + h * 128u;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_f16(d_tmem, umma_desc_sw128(w_addr + h * (W_BYTES / 2) + kk * 32),
                     umma_desc_sw128(tail_addr + kk * 32), idesc_t, (!first_kb || kk != 0) ? 1u : 0u);
        }
      };
      uint32_t use0 = 0, use1 = 0;       // completed uses of each accumulator
      for (uint32_t i = 0; ok; ++i) {
        int L = 0;
        if (!next_tile(sh, i, &L)) break;
        mbar_arrive(&sh->tq_empty[i % TQ]);
        if (L >= total) break;
        const Tile t = decode_tile(L, sh, Gt, tiles_n, BN);
        const bool h0 = t.has0(), h1 = t.has1(), sw = t.swap1();
        if (h0) {
          if (!wait_or_abort(&sh->tempty[0], (use0 & 1u) ^ 1u, sh)) { ok = false; break; }
          tc_fence_after();
        }
        // sub-tile 0 over the first P stages while accumulator 1 may still drain
        const int P = nkb < STAGES ? nkb : STAGES;
        const uint32_t st0 = stage;
        for (int j = 0; j < P; ++j) {
          if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
          if (GATHER) fence_proxy_async();     // the cp.async rows, for the tensor cores' reads
          tc_fence_after();
          if (h0) issue(stage, 0, j == 0);
          if (!h1) umma_commit(&sh->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (h1) {
          if (!wait_or_abort(&sh->tempty[1], (use1 & 1u) ^ 1u, sh)) { ok = false; break; }
          tc_fence_after();
          uint32_t s2 = st0;
          for (int j = 0; j < P; ++j) {
            if (sw) issue_swapped(s2, t.tn, j == 0); else issue(s2, 1, j == 0);
            umma_commit(&sh->empty[s2]);
            if (++s2 == STAGES) s2 = 0;
          }
        }
        for (int kb = P; kb < nkb; ++kb) {
          if (!wait_or_abort(&sh->full[stage], phase, sh)) { ok = false; break; }
          if (GATHER) fence_proxy_async();
          tc_fence_after();
          if (h0) issue(stage, 0, false);
          if (h1) { if (sw) issue_swapped(stage, t.tn, false); else issue(stage, 1, false); }
          umma_commit(&sh->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (h0) { umma_commit(&sh->tfull[0]); ++use0; }
        if (h1) { umma_commit(&sh->tfull[1]); ++use1; }
      }
      // every MMA of this CTA has finished once this barrier flips
      umma_commit(&sh->mma_done);
      mbar_wait(&sh->mma_done, 0);
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> global
    // Each warp copies its 32 lanes x 128 columns of an accumulator into registers
    // behind one wait, releases the accumulator, and only then converts and stores,
    // so the MMA warp waits for the TMEM copy, not for the global stores.
    const int q = warp & 3;                   // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;         // column half (normal) / row or W half (swapped)
    // this warp's output staging box (1024-aligned, for the 64-byte swizzle)
    const uint32_t box = smem_u32(smem + (size_t)STAGES * STAGE_BYTES + kSharedPad) + (warp - 2) * OUT_BOX;
    bool box_busy = false;                    // a TMA store may still be reading the box
    uint32_t use0 = 0, use1 = 0;
    for (uint32_t i = 0;; ++i) {
      // every lane waits (and acquires); the outcome is made warp-uniform
      int L = 0;
      const bool okq = __all_sync(0xffffffffu, next_tile(sh, i, &L));
      if (!okq) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->tq_empty[i % TQ]);
      if (L >= total) break;
      // only the kind here; the rest of the tile is decoded again after the TMEM
      // loads, so it is not held in registers across them
      const int kind = decode_tile(L, sh, Gt, tiles_n, BN).kind;
      bool ok = true;
      for (int sub = 0; sub < 2; ++sub) {
        if (sub == 0 ? kind == K_T : kind == K_SINGLE) continue;
        uint32_t& use = sub == 0 ? use0 : use1;
        if (!__all_sync(0xffffffffu, wait_or_abort(&sh->tfull[sub], use & 1u, sh))) { ok = false; break; }
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + sub * 256u;
        uint32_t v[128];
        const bool swapped = sub == 1 && kind >= K_ST;
        if (MODE == 0) {               // gate columns [64 h, 64 h + 64) and the matching up columns
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_ld16(tbase + half * 64 + 16 * j, v + 16 * j);
            tmem_ld16(tbase + 128 + half * 64 + 16 * j, v + 64 + 16 * j);
          }
        } else {                       // output columns [128 h, 128 h + 128)
#pragma unroll
          for (int j = 0; j < 8; ++j) tmem_ld16(tbase + half * 128 + 16 * j, v + 16 * j);
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tempty[sub]);
        ++use;
        const Tile t = decode_tile(L, sh, Gt, tiles_n, BN);
        if (swapped) {
          store_swapped<MODE>(v, t, half, q, lane, n_out, rows_cap + xg.rows, out);
          continue;
        }
        // 32 rows (one per lane) x NC output columns (gate/up: h = silu(gate) * up of 64
        // hidden units; down: 128 columns of y), as NC / 32 boxes of 32 x 32 through
        // shared memory: lane l writes row l's 64 bytes (16-byte chunk c at slot
        // c ^ ((l >> 1) & 3), the 64-byte swizzle), the warp fences the writes for the
        // TMA engine, and lane 0 stores the box, which the TMA store clips at the
        // output's last row and column
        constexpr int NC = MODE == 0 ? 64 : 128;
        const int row = t.row0 + sub * SUB + q * 32;
#pragma unroll
        for (int cc = 0; cc < NC / 32; ++cc) {
          if (box_busy) {
            if (lane == 0) bulk_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int j = cc * 32 + c * 8;
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              o[i] = MODE == 0 ? silu_f(__uint_as_float(v[j + i])) * __uint_as_float(v[64 + j + i])
                               : __uint_as_float(v[j + i]);
            uint4 pk;
            pk.x = pack_bf16x2(o[0], o[1]); pk.y = pack_bf16x2(o[2], o[3]);
            pk.z = pack_bf16x2(o[4], o[5]); pk.w = pack_bf16x2(o[6], o[7]);
            sts16(box + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), pk);
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, box, t.n0 + half * NC + cc * 32, row);
            bulk_commit();
          }
          box_busy = true;
        }
      }
      if (!ok) break;
    }
    // every output box of this warp is in global memory before the kernel ends
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  // the last CTA to finish puts the launch's tile counter back to 0 (every CTA has
  // stopped claiming by now)
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&ctr[1], 1) == (int)gridDim.x - 1) {
      atomicExch(&ctr[0], 0);
      atomicExch(&ctr[1], 0);
    }
  }
}

// One counter for every launch of either form, so launches in flight on different
// streams never share a tile-counter slot.
static std::atomic<unsigned> g_next_slot{0};

template <int MODE, bool GATHER>
static cudaError_t launch_pass(const CUtensorMap& a, const CUtensorMap& at, const CUtensorMap& b0,
                               const CUtensorMap& b1, const int32_t* offsets, int G, int K, int n_out,
                               int64_t rows_cap, void* out, const int32_t* token_of_row, int T,
                               const void* xsrc, const ExtraGroup& xg, cudaStream_t s) {
  // the output map: rows_cap routed rows, then the extra group's
  CUtensorMap my;
  if (!make_map_bf16_store32(&my, out, (uint64_t)(rows_cap + xg.rows), (uint64_t)n_out))
    return cudaErrorInvalidValue;
  constexpr int BN = MODE == 0 ? 128 : 256;
  const cudaError_t e = ensure_smem_attr((const void*)ffn_tc_kernel<MODE, GATHER>, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (n_out + BN - 1) / BN;
  const int64_t max_tiles = ((rows_cap + xg.rows + SUB - 1) / SUB + G + 1) * tiles_n;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  const int slot = (int)(g_next_slot.fetch_add(1) % kCtrSlots);
  ffn_tc_kernel<MODE, GATHER><<<grid, THREADS, kSmem, s>>>(a, at, b0, b1, offsets, G, K, n_out, rows_cap,
                                                           static_cast<__nv_bfloat16*>(out), slot, token_of_row, T,
                                                           static_cast<const uint8_t*>(xsrc), xg, my);
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_ffn_bf16(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                            const void* w1, const void* w3, const void* w2, int d, int f, void* h,
                            void* y, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > tc::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mx, mxt, m1, m3, mh, mht, m2;
  if (!make_map_bf16(&mx, x_rows, rows_cap, d, tc::SUB) ||
      !make_map_bf16(&mxt, x_rows, rows_cap, d, tc::TAIL_BOX) ||
      !make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) || !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128) ||
      !make_map_bf16(&mh, h, rows_cap, f, tc::SUB) || !make_map_bf16(&mht, h, rows_cap, f, tc::TAIL_BOX) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  tc::ExtraGroup none{};
  none.a = none.at = none.b0 = none.b1 = mx;
  cudaError_t e = tc::launch_pass<0, false>(mx, mxt, m1, m3, offsets, G, d, f, rows_cap, h, nullptr, 0, nullptr, none, s);
  if (e != cudaSuccess) return e;
  return tc::launch_pass<1, false>(mh, mht, m2, m2, offsets, G, f, d, rows_cap, y, nullptr, 0, nullptr, none, s);
}

cudaError_t launch_ffn_bf16_shared(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                                   const void* w1, const void* w3, const void* w2, int d, int f, void* h, void* y,
                                   const void* xs, int Ts, const void* ws1, const void* ws3, const void* ws2,
                                   cudaStream_t s) {
  if (G > tc::kMaxGroups - 1) return cudaErrorInvalidValue;
  if (Ts == 0) return launch_ffn_bf16(x_rows, rows_cap, offsets, G, w1, w3, w2, d, f, h, y, s);
  // h and y hold the groups' rows_cap rows followed by the shared expert's Ts rows;
  // with no routed rows the routed input map points at xs (never read)
  const int64_t hr = rows_cap + Ts;
  const void* xr = rows_cap > 0 ? x_rows : xs;
  const int64_t xrows = rows_cap > 0 ? rows_cap : Ts;
  CUtensorMap mx, mxt, m1, m3, mh, mht, m2;
  tc::ExtraGroup g0{}, g1{};
  if (!make_map_bf16(&mx, xr, xrows, d, tc::SUB) || !make_map_bf16(&mxt, xr, xrows, d, tc::TAIL_BOX) ||
      !make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) || !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128) ||
      !make_map_bf16(&mh, h, hr, f, tc::SUB) || !make_map_bf16(&mht, h, hr, f, tc::TAIL_BOX) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256) || !make_map_bf16(&g0.a, xs, Ts, d, tc::SUB) ||
      !make_map_bf16(&g0.at, xs, Ts, d, tc::TAIL_BOX) || !make_map_bf16(&g0.b0, ws1, f, d, 128) ||
      !make_map_bf16(&g0.b1, ws3, f, d, 128) || !make_map_bf16(&g1.b0, ws2, d, f, 256))
    return cudaErrorInvalidValue;
  g0.a_base = 0;
  g1.a = mh;
  g1.at = mht;
  g1.b1 = g1.b0;
  g1.a_base = (int)rows_cap;
  g0.rows = g1.rows = Ts;
  cudaError_t e = tc::launch_pass<0, false>(mx, mxt, m1, m3, offsets, G, d, f, rows_cap, h, nullptr, 0, nullptr, g0, s);
  if (e != cudaSuccess) return e;
  return tc::launch_pass<1, false>(mh, mht, m2, m2, offsets, G, f, d, rows_cap, y, nullptr, 0, nullptr, g1, s);
}

cudaError_t launch_ffn_bf16_gather(const void* x, int T, const int32_t* token_of_row, int64_t rows_cap,
                                   const int32_t* offsets, int G, const void* w1, const void* w3, const void* w2,
                                   int d, int f, void* h, void* y, const void* ws1, const void* ws3,
                                   const void* ws2, cudaStream_t s) {
  if (G > tc::kMaxGroups - 1) return cudaErrorInvalidValue;
  const int Ts = ws1 ? T : 0;                      // the shared expert over every token, fused
  if (T == 0 || (rows_cap == 0 && Ts == 0) || G == 0) return cudaSuccess;
  // h and y hold the groups' rows_cap rows, then (fused) the shared expert's T rows
  const int64_t hr = rows_cap + Ts;
  CUtensorMap m1, m3, mh, mht, m2;
  tc::ExtraGroup g0{}, g1{};
  if (!make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) || !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128) ||
      !make_map_bf16(&mh, h, hr, f, tc::SUB) || !make_map_bf16(&mht, h, hr, f, tc::TAIL_BOX) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  g0.a = g0.at = g0.b0 = g0.b1 = g1.a = g1.at = g1.b0 = g1.b1 = mh;
  if (Ts > 0) {
    if (!make_map_bf16(&g0.a, x, Ts, d, tc::SUB) || !make_map_bf16(&g0.at, x, Ts, d, tc::TAIL_BOX) ||
        !make_map_bf16(&g0.b0, ws1, f, d, 128) || !make_map_bf16(&g0.b1, ws3, f, d, 128) ||
        !make_map_bf16(&g1.b0, ws2, d, f, 256))
      return cudaErrorInvalidValue;
    g1.a = mh;
    g1.at = mht;
    g1.b1 = g1.b0;
    g1.a_base = (int)rows_cap;
  }
  g0.rows = g1.rows = Ts;
  cudaError_t e = tc::launch_pass<0, true>(mh, mht, m1, m3, offsets, G, d, f, rows_cap, h, token_of_row, T, x, g0, s);
  if (e != cudaSuccess) return e;
  return tc::launch_pass<1, false>(mh, mht, m2, m2, offsets, G, f, d, rows_cap, y, nullptr, 0, nullptr, g1, s);
}

}  // namespace moe
