// The two passes of the bf16 grouped FFN as separate launches (ffn_tc.cu's kernel):
// the first pass alone over some rows, and the second pass with the shared expert's
// rows as one more group, so a caller can run the shared expert's first pass on
// another stream.
#include "common.cuh"
#include "internal.h"

namespace moe {

// The first pass alone: h = silu(x W1^T) * (x W3^T) over the groups' rows.
cudaError_t launch_ffn_bf16_gate_up(const void* x_rows, int64_t rows_cap, const int32_t* offsets, int G,
                                    const void* w1, const void* w3, int d, int f, void* h, cudaStream_t s) {
  if (rows_cap == 0 || G == 0) return cudaSuccess;
  if (G > tc::kMaxGroups) return cudaErrorInvalidValue;
  CUtensorMap mx, mxt, m1, m3;
  if (!make_map_bf16(&mx, x_rows, rows_cap, d, tc::SUB) || !make_map_bf16(&mxt, x_rows, rows_cap, d, tc::TAIL_BOX) ||
      !make_map_bf16(&m1, w1, (uint64_t)G * f, d, 128) || !make_map_bf16(&m3, w3, (uint64_t)G * f, d, 128))
    return cudaErrorInvalidValue;
  tc::ExtraGroup none{};
  none.a = none.at = none.b0 = none.b1 = mx;
  return tc::launch_pass<0, false>(mx, mxt, m1, m3, offsets, G, d, f, rows_cap, h, nullptr, 0, nullptr, none, s);
}

// The second pass alone: y = h W2^T over the groups' rows, and with Ts > 0 the shared
// expert's Ts rows of h after rows_cap through ws2 into y's rows after rows_cap, in
// the same launch (h and y hold rows_cap + Ts rows).
cudaError_t launch_ffn_bf16_down(const void* h, int64_t rows_cap, const int32_t* offsets, int G, const void* w2,
                                 int d, int f, void* y, int Ts, const void* ws2, cudaStream_t s) {
  if (G > tc::kMaxGroups - 1) return cudaErrorInvalidValue;
  const int64_t hr = rows_cap + Ts;
  if (hr == 0 || G == 0) return cudaSuccess;
  CUtensorMap mh, mht, m2;
  if (!make_map_bf16(&mh, h, hr, f, tc::SUB) || !make_map_bf16(&mht, h, hr, f, tc::TAIL_BOX) ||
      !make_map_bf16(&m2, w2, (uint64_t)G * d, f, 256))
    return cudaErrorInvalidValue;
  tc::ExtraGroup g1{};
  g1.a = mh;
  g1.at = mht;
  g1.b0 = g1.b1 = m2;
  if (Ts > 0) {
    if (!make_map_bf16(&g1.b0, ws2, d, f, 256)) return cudaErrorInvalidValue;
    g1.b1 = g1.b0;
    g1.a_base = (int)rows_cap;
  }
  g1.rows = Ts;
  return tc::launch_pass<1, false>(mh, mht, m2, m2, offsets, G, f, d, rows_cap, y, nullptr, 0, nullptr, g1, s);
}

}  // namespace moe
