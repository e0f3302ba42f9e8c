// KV-store step for sm_100a: quantise the step's new tokens' latent to e4m3 with a per-token
// scale and scatter each into its page (the producer of the cache the decode kernel reads).
//
// For new token i of request b at position t = cache_lengths[b] + i, with x its 576 bf16 values:
//   scale = f32(max |x|) / 448, rounded to fp32 (1.0 for an all-zero row),
//   code_d = e4m3_rn_sat(f32_rn(x_d / scale))    (IEEE division, then round-to-nearest-even to
//                                                  e4m3 with saturation to +-448),
// written to blocks[blk, 0, layer, t % P, 0, :] with blk = lookup_table[b][t / P], and the scale to
// scales[sblk, 0, layer, t % P, 0, 0] with sblk from scales_lookup_table when given, else blk
// (the layout of generic_get_paged_cache_with_scales; the quantiser is the pages' data recipe:
// per-token scale amax / 448, e4m3 round-to-nearest with saturation).
//
// Eight lanes per token (a warp stores four tokens): lane k of a token's group reads 16-byte chunks
// k, k + 8, ..., k + 64 of the 1152-byte bf16 row (each step of the group reads 128 contiguous
// bytes), the group reduces |x| with shuffles, and each lane writes the 8 code bytes of each of its
// nine chunks.  HBM-bound: 1152 B read and 580 B written per token.
#pragma once
#include <cstdint>
#include "mla_kernels.cuh"

namespace mla {

struct KvStoreParams {
  const uint16_t* latent;          // bf16 bits [B, T, 576]
  const uint32_t* cache_lengths;   // [B]
  const uint32_t* lut;             // [B, max_pages]
  const uint32_t* slut;            // [B, max_pages] or null
  uint8_t* blocks;                 // e4m3 [NB, KVD, NL, P, 1, 576]
  float* scales;                   // fp32 [NSB, KVD, NL, P, 1, 1]
  unsigned int* status;
  int B, T, P, KVD, NL, layer, NB, NSB, max_pages;
  FastDiv divT;                    // token -> (request, new-token index)
};

constexpr int KVS_WARPS = 8;

// Two fp32 values -> two e4m3 codes (round to nearest even, saturate to the largest finite value);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_rn_sat(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// The quotient x / s is only needed to e4m3 precision.  With r = RN(1 / s), y = RN(x * r) is
// within 2.5 fp32 ulps of RN(x / s) (two roundings of relative size 2^-24 each, plus the half ulp
// of RN(x / s)), so both round to the same e4m3 code unless they straddle a rounding midpoint of
// e4m3: a value whose low 20 mantissa bits are 0x80000 in the normal range (e4m3 keeps 3 of the
// 23 bits), or any value in the subnormal range |y| < 2^-6 (steps of 2^-9).  needs_exact flags y
// within 4 ulps of a midpoint or in that range; only those values take the IEEE division.
__device__ __forceinline__ bool needs_exact(float y) {
  const uint32_t u = __float_as_uint(y);
  return ((u & 0xFFFFFu) - 0x7FFFCu) <= 8u || (fabsf(y) < 0.015625f && y != 0.f);
}

// 8 bf16 (one 16-byte chunk) / s -> 8 e4m3 codes; r = RN(1 / s).
__device__ __forceinline__ uint2 quant8(uint4 v, float s, float r) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  float y[8];
  bool slow = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    y[2 * k] = bf16_lo(in[k]) * r;
    y[2 * k + 1] = bf16_hi(in[k]) * r;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) slow |= needs_exact(y[j]);
  if (slow) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = (j & 1) ? bf16_hi(in[j >> 1]) : bf16_lo(in[j >> 1]);
      if (needs_exact(y[j])) y[j] = __fdiv_rn(x, s);
    }
  }
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) c[k] = e4m3x2_rn_sat(y[2 * k], y[2 * k + 1]);
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ float absmax8(uint4 v, float m) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(in[k])), fabsf(bf16_hi(in[k]))));
  return m;
}

constexpr int KVS_LANES = 8;                       // lanes per token
constexpr int KVS_CHUNKS = 576 * 2 / 16 / KVS_LANES;   // 16-byte bf16 chunks per lane (9)

__global__ void __launch_bounds__(32 * KVS_WARPS) mla_kv_store_kernel(const __grid_constant__ KvStoreParams p) {
  const int lane = threadIdx.x & 31, k = lane & (KVS_LANES - 1);
  const uint32_t tok = (blockIdx.x * blockDim.x + threadIdx.x) / KVS_LANES;
  const bool live = tok < static_cast<uint32_t>(p.B) * static_cast<uint32_t>(p.T);
  bool ok = live;
  size_t row = 0, srow = 0;
  if (live) {
    const uint32_t b = p.divT.div(tok);
    const uint32_t i = tok - b * static_cast<uint32_t>(p.T);
    // destination row (uniform over the token's 8 lanes; a bad id is flagged and the token skipped)
    const uint64_t pos = static_cast<uint64_t>(p.cache_lengths[b]) + i;
    const uint64_t page = pos / static_cast<uint64_t>(p.P);
    const uint32_t slot = static_cast<uint32_t>(pos - page * static_cast<uint64_t>(p.P));
    if (page >= static_cast<uint64_t>(p.max_pages)) {
      ok = false;
    } else {
      const uint32_t blk = p.lut[static_cast<size_t>(b) * p.max_pages + page];
      const uint32_t sblk = p.slut ? p.slut[static_cast<size_t>(b) * p.max_pages + page] : blk;
      ok = blk < static_cast<uint32_t>(p.NB) && sblk < static_cast<uint32_t>(p.NSB);
      row = ((static_cast<size_t>(blk) * p.KVD) * p.NL + p.layer) * p.P + slot;
      srow = ((static_cast<size_t>(sblk) * p.KVD) * p.NL + p.layer) * p.P + slot;
    }
    if (!ok && k == 0) atomicOr(p.status, 1u);
  }
  uint4 v[KVS_CHUNKS];
  float m = 0.f;
  if (ok) {
    const uint4* src = reinterpret_cast<const uint4*>(p.latent + static_cast<size_t>(tok) * 576);
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) v[j] = src[k + KVS_LANES * j];
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) m = absmax8(v[j], m);
  }
  // reduce over the token's 8 lanes (all 32 lanes take part; dead tokens carry m = 0)
#pragma unroll
  for (int o = KVS_LANES / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (!ok) return;
  const float s = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
  const float r = __frcp_rn(s);
  uint2* dst = reinterpret_cast<uint2*>(p.blocks + row * 576);
#pragma unroll
  for (int j = 0; j < KVS_CHUNKS; ++j) dst[k + KVS_LANES * j] = quant8(v[j], s, r);
  if (k == 0) p.scales[srow] = s;
}

}  // namespace mla
