// LSE merge of partial decode results (sm_100a): the combine step of context parallelism, where
// each rank decodes a contiguous page range of every request's keys and the ranks' results are
// merged after an exchange.  For a row (request, query token, head) with parts r = 0..R-1:
//   lse = ln sum_r e^{lse_r},   out = sum_r e^{lse_r - lse} out_r
// (the softmax over the union of the key ranges, written from the parts' normalised results and
// their log-sum-exps).  A part with lse = -inf has no keys and is skipped; a row whose parts are all
// empty gets out = 0 and lse = -inf.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace mla {

constexpr int MERGE_WARPS = 8;

// One warp per row (grid-stride); lane l handles the 16 values [16 l, 16 l + 16) of the 512.
__global__ void __launch_bounds__(32 * MERGE_WARPS)
mla_merge_parts_kernel(const uint16_t* __restrict__ outs, const float* __restrict__ lses, int R, long long rows,
                       uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const long long stride = static_cast<long long>(gridDim.x) * MERGE_WARPS;
  for (long long row = static_cast<long long>(blockIdx.x) * MERGE_WARPS + (threadIdx.x >> 5); row < rows;
       row += stride) {
    float mx = -INFINITY, tot = 0.f, acc[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) acc[x] = 0.f;
    for (int r = 0; r < R; ++r) {
      const float l = lses[static_cast<long long>(r) * rows + row];
      if (l == -INFINITY) continue;
      const uint4* src = reinterpret_cast<const uint4*>(outs + (static_cast<long long>(r) * rows + row) * 512) + 2 * lane;
      const uint4 a = src[0], b = src[1];
      const uint32_t wds[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      const float mn = fmaxf(mx, l);
      const float sa = __expf(mx - mn), w = __expf(l - mn);     // sa = 0 for the first part
      mx = mn;
      tot = tot * sa + w;
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        acc[2 * x] = acc[2 * x] * sa + w * __uint_as_float(wds[x] << 16);
        acc[2 * x + 1] = acc[2 * x + 1] * sa + w * __uint_as_float(wds[x] & 0xFFFF0000u);
      }
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    uint32_t o[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) o[x] = ptx::pack_bf16x2(acc[2 * x] * inv, acc[2 * x + 1] * inv);
    uint4* dst = reinterpret_cast<uint4*>(out + row * 512) + 2 * lane;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    if (lane == 0 && lse) lse[row] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
  }
}

}  // namespace mla
