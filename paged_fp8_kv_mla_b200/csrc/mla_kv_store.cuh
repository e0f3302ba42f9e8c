// KV-store step for sm_100a: quantise the step's new tokens' latent to e4m3 with a per-token
// scale and scatter each into its page (the producer of the cache the decode kernel reads).
//
// For new token i of request b at position t = cache_lengths[b] + i, with x its 576 bf16 values:
//   scale = f32(max |x|) / 448, rounded to fp32 (1.0 for an all-zero row),
//   code_d = e4m3_rn_sat(f32_rn(x_d / scale))    (IEEE division, then round-to-nearest-even to
//                                                  e4m3 with saturation to +-448),
// written to blocks[blk, 0, layer, t % P, 0, :] with blk = lookup_table[b][t / P], and the scale to
// scales[sblk, 0, layer, t % P, 0, 0] with sblk from scales_lookup_table when given, else blk
// (the layout of generic_get_paged_cache_with_scales; the quantiser is the usual per-token FP8
// recipe, also used to generate the test workloads: scale amax / 448, e4m3 round-to-nearest with
// saturation).
//
// Eight lanes per token (a warp stores four tokens): lane k of a token's group reads 16-byte chunks
// k, k + 8, ..., k + 64 of the 1152-byte bf16 row (each step of the group reads 128 contiguous
// bytes), the group reduces max |x| with shuffles, and each lane writes the 8 code bytes of each of
// its nine chunks.  HBM-bound: 1152 B read and 580 B written per token.
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

// The quotient RN(x / s) by one correction of the reciprocal product (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// with r = RN(1 / s) and y0 = RN(x * r), the remainder x - y0 * s is computed by one fma and
// y = RN(y0 + (x - y0 * s) * r) by another.  Checked in exact arithmetic before use: for bf16 x
// with |x| >= 2^-100 and fp32 s, y equals the IEEE quotient bit for bit (27 M cases); smaller |x|
// (where the remainder can fall into the subnormal range) only reach e4m3 code 0, and for every
// s >= 2^-90 the e4m3 code of y equals the code of RN(x / s) (30 M cases, zeros of both signs
// included).  The remainder is formed as -(y0 * s - x) so that a zero keeps its sign.  Tokens whose
// scale is below 2^-90 take the IEEE division.
constexpr float KVS_FAST_MIN_SCALE = 8.077935669463161e-28f;   // 2^-90

// 8 bf16 (one 16-byte chunk) / s -> 8 e4m3 codes; r = RN(1 / s), s >= 2^-90.
__device__ __forceinline__ uint2 quant8(uint4 v, float s, float r) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  const float2 ss = make_float2(s, s), rr = make_float2(r, r);
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 x = make_float2(bf16_lo(in[k]), bf16_hi(in[k]));
    const float2 y0 = __fmul2_rn(x, rr);
    const float2 t = __ffma2_rn(y0, ss, make_float2(-x.x, -x.y));          // y0 * s - x
    const float2 y = __ffma2_rn(make_float2(-t.x, -t.y), rr, y0);          // y0 + (x - y0 * s) * r
    c[k] = e4m3x2_rn_sat(y.x, y.y);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// The same with the IEEE division (tokens with a scale below 2^-90).
__device__ __forceinline__ uint2 quant8_div(uint4 v, float s) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) c[k] = e4m3x2_rn_sat(__fdiv_rn(bf16_lo(in[k]), s), __fdiv_rn(bf16_hi(in[k]), s));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// max |x| over a chunk as bf16 bit patterns: for non-NaN values the magnitude bits order like the
// magnitudes, so a per-halfword unsigned max of (bits & 0x7FFF) is the bf16 of max |x|.
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v, uint32_t m2) {
  m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
  m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
  m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
  return __vmaxu2(m2, v.w & 0x7FFF7FFFu);
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
  uint32_t m2 = 0;
  if (ok) {
    const uint4* src = reinterpret_cast<const uint4*>(p.latent + static_cast<size_t>(tok) * 576);
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) v[j] = src[k + KVS_LANES * j];
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) m2 = absmax8_bits(v[j], m2);
  }
  // reduce over the token's 8 lanes (all 32 lanes take part; dead tokens carry 0)
#pragma unroll
  for (int o = KVS_LANES / 2; o > 0; o >>= 1) m2 = __vmaxu2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  if (!ok) return;
  const float m = __uint_as_float(max(m2 & 0xFFFFu, m2 >> 16) << 16);
  const float s = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
  uint2* dst = reinterpret_cast<uint2*>(p.blocks + row * 576);
  if (s >= KVS_FAST_MIN_SCALE) {
    const float r = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) dst[k + KVS_LANES * j] = quant8(v[j], s, r);
  } else {
#pragma unroll
    for (int j = 0; j < KVS_CHUNKS; ++j) dst[k + KVS_LANES * j] = quant8_div(v[j], s);
  }
  if (k == 0) p.scales[srow] = s;
}

}  // namespace mla
