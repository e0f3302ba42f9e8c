// Device code of the paged FP8-KV MLA decode for sm_100a.
//
// Work decomposition.  An "item" is one (request b, query token i, group of 128
// query heads g).  Item keys are tiled in BN = 64-token tiles; all items' tiles
// are laid end to end and cut into equal contiguous ranges, one per 2-CTA
// cluster.  A cluster walks the pieces ("units") of items that fall in its
// range.  An item cut by a range boundary is "split": each piece writes a
// normalised fp32 partial and its LSE, and the combine kernel merges them.
//
// Inside a cluster the two CTAs split the 576 latent dims: CTA c owns latent
// dims [256c, 256c+256) and rope dims [512+32c, 512+32c+32), i.e. half of every
// token's bytes.  Each CTA computes a partial Q.K^T over its 288 dims with
// tcgen05 MMAs (M = 128 heads), the two partial score tiles are exchanged
// through distributed shared memory and added, both CTAs run the same online
// softmax, and each computes P.V for its own 256 V dims (V = the first 512
// latent dims).  TMEM per CTA: O 128 x 256 fp32 (cols 0..255) and two score
// buffers of 64 cols (P overwrites its score buffer as packed bf16).
//
// Warp roles per CTA (320 threads):
//   warps 0-3  converter: Q tile load at each unit start; FP8 -> bf16 dequant of
//              every KV tile into the UMMA K-major SWIZZLE_128B/64B layout
//   warps 4-7  softmax: score exchange, online softmax, P -> TMEM, O rescale,
//              epilogue (one thread per head row / TMEM lane)
//   warp 8     producer: TMA loads of the FP8 rows + bulk copies of the scales
//   warp 9     MMA issuer (lane 0) and TMEM owner
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"

namespace mla {

constexpr int BN = 64;          // tokens per tile
constexpr int HEAD_DIM = 576;
constexpr int V_DIM = 512;
constexpr int MROWS = 128;      // query heads per item (MMA M)
constexpr int NUM_THREADS = 320;
constexpr int NFP8 = 2;         // FP8 staging stages

// ---- shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SQ_LAT = 0;            // Q latent half: 4 atom columns x (128 rows x 128 B), SW128
constexpr uint32_t SQ_ROPE = 65536;       // Q rope half: 128 rows x 64 B, SW64
constexpr uint32_t SK0 = 73728;           // bf16 K tiles (2): latent 4 x (64 x 128 B) SW128, rope 64 x 64 B SW64
constexpr uint32_t SK_STRIDE = 36864;
constexpr uint32_t SK_ROPE = 32768;
constexpr uint32_t SF0 = SK0 + 2 * SK_STRIDE;   // FP8 stages
constexpr uint32_t SF_STRIDE = 19456;
constexpr uint32_t SF_ROPE = 16384;       // 64 rows x 32 B
constexpr uint32_t SF_SC = 18432;         // 64 fp32 scales
// partial-score exchange: [16 chunks][128 rows][16 B], so that one warp-wide store of chunk v by
// 32 consecutive rows is 512 contiguous bytes
constexpr uint32_t SX = SF0 + NFP8 * SF_STRIDE;
constexpr uint32_t SX_CHUNK = MROWS * 16;
constexpr uint32_t SBAR = SX + 16 * SX_CHUNK;
constexpr uint32_t SMEM_USED = SBAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;   // slack for aligning the base

// barrier indices (8 bytes each from SBAR)
enum Bar : uint32_t {
  B_FP8_FULL = 0, B_FP8_EMPTY = 2, B_K_FULL = 4, B_K_EMPTY = 6, B_S_FULL = 8, B_P_FULL = 10,
  B_O_DONE = 12, B_O_FREE = 14, B_Q_FULL = 15, B_Q_FREE = 16, B_XS_FULL = 17, B_XS_FREE = 18,
  B_DRAIN = 19, NUM_BARS = 20
};
constexpr uint32_t S_TMEM_BASE = SBAR + 256;
constexpr uint32_t S_ABORT = SBAR + 260;

// TMEM columns
constexpr uint32_t T_O = 0;
constexpr uint32_t T_S = 256;             // + 64 * buffer
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(128, BN, false, false);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, 256, false, true);

constexpr unsigned STATUS_BOUNDS = 1u;
constexpr unsigned STATUS_TIMEOUT = 2u;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait

// Optional per-stage timestamps (build with -DMLA_TRACE): cluster 0 writes %clock64 values
// to trace[(cta * TRACE_TILES + tile) * TRACE_EVENTS + event] for its first TRACE_TILES tiles.
constexpr int TRACE_TILES = 64;
constexpr int TRACE_EVENTS = 32;

struct DecodeParams {
  unsigned long long* trace;       // null unless tracing
  const uint16_t* q;               // bf16 bits [B, T, H, 576]
  const float* scales;
  const int32_t* item_start;       // [items + 1] tile prefix
  const int32_t* item_nvis;        // [items] visible keys (clamped)
  const int32_t* cluster_first;    // [NC] first item of each cluster range
  const int32_t* hdr;              // [0] tiles per cluster, [1] total tiles
  const uint32_t* lut;
  const uint32_t* slut;            // may be null
  uint16_t* out;                   // bf16 bits [B, T, H, 512]
  float* lse;                      // may be null
  float* part_o;                   // [2 NC][128][512]
  float* part_lse;                 // [2 NC][128]
  unsigned int* status;
  int B, T, H, G, P, KVD, NL, layer, NB, NSB, max_pages, boxr, items, NC;
  float scale_log2;                // softmax_scale * log2(e)
};

struct Unit {
  int item, b, i, g, nvis;
  int tb, te;       // tile range within the item
  int slot;         // partial slot, -1 = write out directly
};

// Walks the units of cluster `k`: the pieces of items inside tile range [R0, R1).
struct UnitWalker {
  const DecodeParams& p;
  int k, R0, R1, it;
  __device__ UnitWalker(const DecodeParams& p_, int k_) : p(p_), k(k_) {
    const int tpc = p.hdr[0], total = p.hdr[1];
    R0 = k * tpc;
    R1 = min(total, R0 + tpc);
    it = p.cluster_first[k];
  }
  __device__ bool next(Unit& u) {
    if (R0 >= R1 || it >= p.items) return false;
    const int s = p.item_start[it], e = p.item_start[it + 1];
    const int a = max(s, R0), z = min(e, R1);
    if (a >= z) return false;
    u.item = it;
    u.g = it % p.G;
    u.i = (it / p.G) % p.T;
    u.b = it / (p.G * p.T);
    u.nvis = p.item_nvis[it];
    u.tb = a - s;
    u.te = z - s;
    const bool split = (s < R0) || (e > R1);
    u.slot = split ? (2 * k + (a == R0 ? 0 : 1)) : -1;
    ++it;
    return true;
  }
};

#ifdef MLA_TRACE
#define MLA_TRACE_EV(tile, ev)                                                                        \
  do {                                                                                                \
    if (p.trace && k == 0 && (tile) < static_cast<uint32_t>(TRACE_TILES))                            \
      p.trace[(c * TRACE_TILES + (tile)) * TRACE_EVENTS + (ev)] = clock64();                         \
  } while (0)
#else
#define MLA_TRACE_EV(tile, ev) do {} while (0)
#endif

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(uint32_t i) const { return base + SBAR + 8 * i; }
};

__device__ __forceinline__ volatile uint32_t* abort_flag(uint8_t* smem_base) {
  return reinterpret_cast<volatile uint32_t*>(smem_base + S_ABORT);
}

__device__ unsigned int g_status_word;   // sticky device status (bit 0 bounds, bit 1 timeout)

__device__ __forceinline__ void raise_status(unsigned int* status, unsigned bits) {
  atomicOr(status ? status : &g_status_word, bits);
}

// Bounded wait on an mbarrier phase (slow path below).  Returns false (and marks the CTA, its peer and the
// status word) when the wait gives up or another role already gave up.
__device__ __noinline__ bool wait_bar_slow(uint32_t addr, uint32_t parity, bool cluster_scope,
                                           volatile uint32_t* abort, unsigned int* status, uint32_t peer_abort) {
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
    for (int i = 0; i < 256; ++i) {
      if (cluster_scope ? ptx::mbar_try_wait_relaxed_cluster(addr, parity) : ptx::mbar_try_wait(addr, parity)) {
        if (cluster_scope) ptx::fence_acq_rel_cluster();
        return true;
      }
    }
    if (*abort) return false;
    if (ptx::globaltimer() - t0 > WAIT_LIMIT_NS) {
      *abort = 1u;
      if (peer_abort) ptx::st_cluster_u32(peer_abort, 1u);
      raise_status(status, STATUS_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ bool wait_bar(uint32_t addr, uint32_t parity, bool cluster_scope, volatile uint32_t* abort,
                                         unsigned int* status, uint32_t peer_abort) {
  if (cluster_scope) {
    if (ptx::mbar_try_wait_relaxed_cluster(addr, parity)) {
      ptx::fence_acq_rel_cluster();
      return true;
    }
  } else if (ptx::mbar_try_wait(addr, parity)) {
    return true;
  }
  return wait_bar_slow(addr, parity, cluster_scope, abort, status, peer_abort);
}

// ---------------------------------------------------------------------------------------------
// Producer: issue the loads of one 64-token tile of request b starting at token tok0 (nv valid
// rows) into one FP8 stage, completing on `full`.  Rows are loaded in boxes of `boxr` rows, each
// inside one page; boxes whose page id is out of range are skipped and flagged.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ bool box_source(const DecodeParams& p, int b, int tok, uint32_t& row, uint32_t& srow) {
  const int page = tok / p.P;
  const int slot = tok - page * p.P;
  if (page >= p.max_pages) return false;
  const uint32_t blk = p.lut[static_cast<size_t>(b) * p.max_pages + page];
  const uint32_t sblk = p.slut ? p.slut[static_cast<size_t>(b) * p.max_pages + page] : blk;
  if (blk >= static_cast<uint32_t>(p.NB) || sblk >= static_cast<uint32_t>(p.NSB)) return false;
  row = ((blk * static_cast<uint32_t>(p.KVD)) * p.NL + p.layer) * p.P + slot;
  srow = ((sblk * static_cast<uint32_t>(p.KVD)) * p.NL + p.layer) * p.P + slot;
  return true;
}

__device__ __forceinline__ void produce_tile(const DecodeParams& p, const CUtensorMap* tm_lat,
                                             const CUtensorMap* tm_rope, int c, int b, int tok0, int nv,
                                             uint32_t stage, uint32_t full) {
  uint32_t bytes = 0;
  bool bad = false;
  for (int r = 0; r < nv; r += p.boxr) {
    uint32_t row, srow;
    if (box_source(p, b, tok0 + r, row, srow)) bytes += p.boxr * (256 + 32 + 4);
    else bad = true;
  }
  if (bad) raise_status(p.status, STATUS_BOUNDS);
  ptx::mbar_arrive_expect_tx(full, bytes);
  for (int r = 0; r < nv; r += p.boxr) {
    uint32_t row, srow;
    if (!box_source(p, b, tok0 + r, row, srow)) continue;
    ptx::tma_load_2d(stage + r * 256, tm_lat, 256 * c, static_cast<int32_t>(row), full);
    ptx::tma_load_2d(stage + SF_ROPE + r * 32, tm_rope, 512 + 32 * c, static_cast<int32_t>(row), full);
    ptx::bulk_load(stage + SF_SC + r * 4, p.scales + srow, p.boxr * 4, full);
  }
}

// ---------------------------------------------------------------------------------------------
// Converter: 16 e4m3 bytes of one row times the row's scale -> 16 bf16 (8 packed words).
// bf16_rn(f32_rn(e4m3 * s)): the e4m3 -> f16 -> f32 steps are exact, the multiply rounds to
// nearest in fp32, the pack rounds to nearest-even bf16.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void dequant16(uint4 raw, float s, uint32_t (&w)[8]) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t h0 = ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] & 0xFFFFu));
    const uint32_t h1 = ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] >> 16));
    const float f0 = ptx::mul_rn(ptx::f16_lo_to_f32(h0), s);
    const float f1 = ptx::mul_rn(ptx::f16_hi_to_f32(h0), s);
    const float f2 = ptx::mul_rn(ptx::f16_lo_to_f32(h1), s);
    const float f3 = ptx::mul_rn(ptx::f16_hi_to_f32(h1), s);
    w[2 * k] = ptx::pack_bf16x2(f0, f1);
    w[2 * k + 1] = ptx::pack_bf16x2(f2, f3);
  }
}

// Byte offset of 16-byte unit `u` (0..7) of row `r` in a K-major SWIZZLE_128B region whose
// 8-row groups are 1024 B apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int u) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4);
}
// Same for SWIZZLE_64B (64-byte rows, 8-row groups 512 B apart, units 0..3).
__device__ __forceinline__ uint32_t sw64_off(int r, int u) {
  return (r >> 3) * 512 + (r & 7) * 64 + ((u ^ ((r & 7) >> 1)) << 4);
}

// Convert one FP8 stage (this CTA's 288 dims of 64 rows) into a bf16 K tile; rows >= nv become 0.
// Called by 128 threads (t = 0..127).
__device__ __forceinline__ void convert_tile(int t, uint32_t stage, uint32_t ktile, int nv) {
  uint4 raw[9];
  float sc[9];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int id = it * 128 + t;
    const int row = id >> 4, cc = id & 15;
    raw[it] = ptx::ld_shared_v4(stage + row * 256 + cc * 16);
    sc[it] = ptx::ld_shared_f32(stage + SF_SC + row * 4);
  }
  raw[8] = ptx::ld_shared_v4(stage + SF_ROPE + (t >> 1) * 32 + (t & 1) * 16);
  sc[8] = ptx::ld_shared_f32(stage + SF_SC + (t >> 1) * 4);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int id = it * 128 + t;
    const int row = id >> 4, cc = id & 15;
    uint32_t w[8];
    dequant16(raw[it], sc[it], w);
    if (row >= nv) {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
    const uint32_t base = ktile + (cc >> 2) * 8192;
    const int u0 = (cc & 3) * 2;
    ptx::st_shared_v4(base + sw128_off(row, u0), w[0], w[1], w[2], w[3]);
    ptx::st_shared_v4(base + sw128_off(row, u0 + 1), w[4], w[5], w[6], w[7]);
  }
  {
    const int row = t >> 1, cc = t & 1;
    uint32_t w[8];
    dequant16(raw[8], sc[8], w);
    if (row >= nv) {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
    const uint32_t base = ktile + SK_ROPE;
    ptx::st_shared_v4(base + sw64_off(row, cc * 2), w[0], w[1], w[2], w[3]);
    ptx::st_shared_v4(base + sw64_off(row, cc * 2 + 1), w[4], w[5], w[6], w[7]);
  }
}

// Q rows of one item, this CTA's 288 dims, into the SW128 / SW64 K-major layout. Rows >= H are 0.
__device__ __forceinline__ void load_q(const DecodeParams& p, const Unit& u, int c, int t, uint32_t sq) {
  const uint16_t* qrow0 = p.q + (static_cast<size_t>(u.b) * p.T + u.i) * p.H * HEAD_DIM;
  const int h0 = u.g * MROWS;
#pragma unroll 1
  for (int batch = 0; batch < 3; ++batch) {
    uint4 v[12];
#pragma unroll
    for (int k = 0; k < 12; ++k) {
      const int id = (batch * 12 + k) * 128 + t;
      const int row = id / 36, cc = id - row * 36;
      const int col = cc < 32 ? 256 * c + cc * 8 : 512 + 32 * c + (cc - 32) * 8;
      v[k] = make_uint4(0, 0, 0, 0);
      if (h0 + row < p.H)
        v[k] = __ldg(reinterpret_cast<const uint4*>(qrow0 + static_cast<size_t>(h0 + row) * HEAD_DIM + col));
    }
#pragma unroll
    for (int k = 0; k < 12; ++k) {
      const int id = (batch * 12 + k) * 128 + t;
      const int row = id / 36, cc = id - row * 36;
      const uint32_t dst = cc < 32 ? sq + SQ_LAT + (cc >> 3) * 16384 + sw128_off(row, cc & 7)
                                   : sq + SQ_ROPE + sw64_off(row, cc - 32);
      ptx::st_shared_v4(dst, v[k].x, v[k].y, v[k].z, v[k].w);
    }
  }
}

// =============================================================================================
// decode kernel
// =============================================================================================
__global__ void __launch_bounds__(NUM_THREADS, 1)
mla_decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tm_lat,
                  const __grid_constant__ CUtensorMap tm_rope) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Smem S{ptx::smem_u32(smem)};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = ptx::cluster_ctarank();
  const uint32_t peer = c ^ 1u;
  const int k = static_cast<int>(ptx::cluster_id_x());
  volatile uint32_t* abort = abort_flag(smem);
  const uint32_t peer_abort = ptx::mapa(S.base + S_ABORT, peer);

  if (threadIdx.x == 0) {
    ptx::mbar_init(S.bar(B_FP8_FULL + 0), 1);
    ptx::mbar_init(S.bar(B_FP8_FULL + 1), 1);
    ptx::mbar_init(S.bar(B_FP8_EMPTY + 0), 128);
    ptx::mbar_init(S.bar(B_FP8_EMPTY + 1), 128);
    ptx::mbar_init(S.bar(B_K_FULL + 0), 128);
    ptx::mbar_init(S.bar(B_K_FULL + 1), 128);
    ptx::mbar_init(S.bar(B_K_EMPTY + 0), 1);
    ptx::mbar_init(S.bar(B_K_EMPTY + 1), 1);
    ptx::mbar_init(S.bar(B_S_FULL + 0), 1);
    ptx::mbar_init(S.bar(B_S_FULL + 1), 1);
    ptx::mbar_init(S.bar(B_P_FULL + 0), 128);
    ptx::mbar_init(S.bar(B_P_FULL + 1), 128);
    ptx::mbar_init(S.bar(B_O_DONE + 0), 1);
    ptx::mbar_init(S.bar(B_O_DONE + 1), 1);
    ptx::mbar_init(S.bar(B_O_FREE), 128);
    ptx::mbar_init(S.bar(B_Q_FULL), 128);
    ptx::mbar_init(S.bar(B_Q_FREE), 1);
    ptx::mbar_init(S.bar(B_XS_FULL), 128);
    ptx::mbar_init(S.bar(B_XS_FREE), 128);
    ptx::mbar_init(S.bar(B_DRAIN), 1);
    *abort = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    ptx::prefetch_tmap(&tm_lat);
    ptx::prefetch_tmap(&tm_rope);
  }
  if (warp == 9) {
    ptx::tmem_alloc(S.base + S_TMEM_BASE, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  ptx::cluster_sync();   // the peer's barriers exist before any remote arrive
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + S_TMEM_BASE);

// Single-thread roles bail out alone; whole-warp roles bail out together so that the
// warp-collective tcgen05 instructions after a wait never run on a partial warp.
#define MLA_WAIT(bar, parity, cl)                                                    \
  if (!wait_bar((bar), (parity), (cl), abort, p.status, peer_abort)) goto role_done;
#define MLA_WAIT_WARP(bar, parity, cl)                                               \
  if (!__all_sync(0xffffffffu, wait_bar((bar), (parity), (cl), abort, p.status, peer_abort))) goto role_done;

  if (warp < 4) {
    // ------------------------------------------------------------------ converter
    const int t = threadIdx.x;
    UnitWalker wk(p, k);
    Unit u;
    uint32_t g = 0, uu = 0;
    while (wk.next(u)) {
      MLA_WAIT_WARP(S.bar(B_Q_FREE), (uu & 1) ^ 1, false);
      if (t == 0) MLA_TRACE_EV(g, 3);
      load_q(p, u, c, t, S.base);
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(S.bar(B_Q_FULL));
      if (t == 0) MLA_TRACE_EV(g, 4);
      for (int j = u.tb; j < u.te; ++j, ++g) {
        const uint32_t s = g & 1, ph = (g >> 1) & 1;
        MLA_WAIT_WARP(S.bar(B_FP8_FULL + s), ph, false);
        if (t == 0) MLA_TRACE_EV(g, 0);
        MLA_WAIT_WARP(S.bar(B_K_EMPTY + s), ph ^ 1, false);
        if (t == 0) MLA_TRACE_EV(g, 1);
        const int nv = min(BN, u.nvis - j * BN);
        convert_tile(t, S.base + SF0 + s * SF_STRIDE, S.base + SK0 + s * SK_STRIDE, nv);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(S.bar(B_FP8_EMPTY + s));
        ptx::mbar_arrive(S.bar(B_K_FULL + s));
        if (t == 0) MLA_TRACE_EV(g, 2);
      }
      ++uu;
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int h = threadIdx.x - 128;
    const int quad = warp - 4;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t xrow_local = S.base + SX + h * 16;
    const uint32_t xrow_peer = ptx::mapa(xrow_local, peer);
    const uint32_t xs_full_peer = ptx::mapa(S.bar(B_XS_FULL), peer);
    const uint32_t xs_free_peer = ptx::mapa(S.bar(B_XS_FREE), peer);
    UnitWalker wk(p, k);
    Unit u;
    uint32_t g = 0, e = 0;
    while (wk.next(u)) {
      float m_ref = -INFINITY, l = 0.f;
      for (int j = u.tb; j < u.te; ++j, ++g, ++e) {
        const uint32_t sb = g & 1;
        MLA_WAIT_WARP(S.bar(B_S_FULL + sb), (g >> 1) & 1, false);
        if (h == 0) MLA_TRACE_EV(g, 8);
        ptx::tc_fence_after();
        float x[BN];
        {
          uint32_t r[32];
          ptx::tmem_ld32(lane_base + T_S + 64 * sb, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = __uint_as_float(r[q]);
          ptx::tmem_ld32(lane_base + T_S + 64 * sb + 32, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) x[32 + q] = __uint_as_float(r[q]);
        }
        if (h == 0) MLA_TRACE_EV(g, 9);
        // exchange partial scores with the peer CTA (it holds the other 288 dims)
        MLA_WAIT_WARP(S.bar(B_XS_FREE), (e & 1) ^ 1, true);
        if (h == 0) MLA_TRACE_EV(g, 10);
#pragma unroll
        for (int v = 0; v < 16; ++v)
          ptx::st_cluster_v4(xrow_peer + v * SX_CHUNK, x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
        ptx::mbar_arrive_remote(xs_full_peer);
        if (h == 0) MLA_TRACE_EV(g, 11);
        MLA_WAIT_WARP(S.bar(B_XS_FULL), e & 1, true);
        if (h == 0) MLA_TRACE_EV(g, 12);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const uint4 o = ptx::ld_shared_v4(xrow_local + v * SX_CHUNK);
          x[4 * v] += __uint_as_float(o.x);
          x[4 * v + 1] += __uint_as_float(o.y);
          x[4 * v + 2] += __uint_as_float(o.z);
          x[4 * v + 3] += __uint_as_float(o.w);
        }
        ptx::mbar_arrive_remote(xs_free_peer);
        if (h == 0) MLA_TRACE_EV(g, 13);
        // online softmax in the log2 domain
        const int nv = min(BN, u.nvis - j * BN);
        float mt = -INFINITY;
#pragma unroll
        for (int q = 0; q < BN; ++q) {
          x[q] = (q < nv) ? x[q] * p.scale_log2 : -INFINITY;
          mt = fmaxf(mt, x[q]);
        }
        float alpha = 1.f;
        bool rescale = false;
        if (mt > m_ref + 8.f) {           // lazy max: keep the reference unless it grows by > 2^8
          const float m_new = mt;
          alpha = (m_ref == -INFINITY) ? 0.f : ptx::ex2_approx(m_ref - m_new);
          l *= alpha;
          rescale = (j != u.tb);
          m_ref = m_new;
        }
        float lsum = 0.f;
        uint32_t pw[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float p0 = ptx::ex2_approx(x[2 * q] - m_ref);
          const float p1 = ptx::ex2_approx(x[2 * q + 1] - m_ref);
          lsum += p0 + p1;
          pw[q] = ptx::pack_bf16x2(p0, p1);
        }
        l += lsum;
        ptx::tmem_st32(lane_base + T_S + 64 * sb, pw);
        // the O rescale uses warp-collective TMEM access: a warp rescales when any of its rows
        // moved its reference max (rows that did not move have alpha == 1)
        if (!rescale) alpha = 1.f;
        if (__any_sync(0xffffffffu, rescale)) {
          const uint32_t gp = g - 1;
          MLA_WAIT_WARP(S.bar(B_O_DONE + (gp & 1)), (gp >> 1) & 1, false);
          ptx::tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t r[32];
            ptx::tmem_ld32(lane_base + T_O + 32 * ch, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
            ptx::tmem_st32(lane_base + T_O + 32 * ch, r);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(S.bar(B_P_FULL + sb));
        if (h == 0) MLA_TRACE_EV(g, 14);
      }
      // epilogue: O / l
      {
        const uint32_t gl = g - 1;
        MLA_WAIT_WARP(S.bar(B_O_DONE + (gl & 1)), (gl >> 1) & 1, false);
        ptx::tc_fence_after();
        const float inv_l = 1.f / l;
        const int head = u.g * MROWS + h;
        const bool row_ok = head < p.H;
        const float lse_v = (m_ref + ptx::lg2_approx(l)) * 0.69314718055994530942f;
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t r[32];
          ptx::tmem_ld32(lane_base + T_O + 32 * ch, r);
          ptx::tmem_wait_ld();
          if (!row_ok) continue;
          if (u.slot < 0) {
            uint16_t* dst = p.out + ((static_cast<size_t>(u.b) * p.T + u.i) * p.H + head) * V_DIM + 256 * c + 32 * ch;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = ptx::pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv_l, __uint_as_float(r[8 * v + 1]) * inv_l);
              w.y = ptx::pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv_l, __uint_as_float(r[8 * v + 3]) * inv_l);
              w.z = ptx::pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv_l, __uint_as_float(r[8 * v + 5]) * inv_l);
              w.w = ptx::pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv_l, __uint_as_float(r[8 * v + 7]) * inv_l);
              reinterpret_cast<uint4*>(dst)[v] = w;
            }
          } else {
            float* dst = p.part_o + (static_cast<size_t>(u.slot) * MROWS + h) * V_DIM + 256 * c + 32 * ch;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              float4 w = make_float4(__uint_as_float(r[4 * v]) * inv_l, __uint_as_float(r[4 * v + 1]) * inv_l,
                                     __uint_as_float(r[4 * v + 2]) * inv_l, __uint_as_float(r[4 * v + 3]) * inv_l);
              reinterpret_cast<float4*>(dst)[v] = w;
            }
          }
        }
        if (c == 0 && row_ok) {
          if (u.slot < 0) {
            if (p.lse) p.lse[(static_cast<size_t>(u.b) * p.T + u.i) * p.H + head] = lse_v;
          } else {
            p.part_lse[static_cast<size_t>(u.slot) * MROWS + h] = lse_v;
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(S.bar(B_O_FREE));
        if (h == 0) MLA_TRACE_EV(g - 1, 15);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      UnitWalker wk(p, k);
      Unit u;
      uint32_t g = 0;
      bool ok = true;
      while (ok && wk.next(u)) {
        for (int j = u.tb; j < u.te; ++j) {
          const uint32_t s = g & 1, ph = (g >> 1) & 1;
          if (!wait_bar(S.bar(B_FP8_EMPTY + s), ph ^ 1, false, abort, p.status, peer_abort)) {
            ok = false;
            break;
          }
          MLA_TRACE_EV(g, 16);
          const int nv = min(BN, u.nvis - j * BN);
          produce_tile(p, &tm_lat, &tm_rope, static_cast<int>(c), u.b, j * BN, nv, S.base + SF0 + s * SF_STRIDE,
                       S.bar(B_FP8_FULL + s));
          MLA_TRACE_EV(g, 17);
          ++g;
        }
      }
      // drain: every issued stage has landed before the CTA may exit
      for (uint32_t d = (g >= 2 ? g - 2 : 0); d < g; ++d) {
        const uint32_t s = d & 1, ph = (d >> 1) & 1;
        if (!ptx::mbar_try_wait(S.bar(B_FP8_FULL + s), ph)) {
          const uint64_t t0 = ptx::globaltimer();
          while (!ptx::mbar_try_wait(S.bar(B_FP8_FULL + s), ph) && ptx::globaltimer() - t0 < WAIT_LIMIT_NS) {}
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      UnitWalker wk(p, k);
      Unit u;
      uint32_t g = 0, uu = 0;
      bool have_prev = false, prev_first = false;
      uint32_t prev_g = 0, prev_u = 0;
      auto issue_pv = [&](uint32_t hg, bool first, uint32_t hu) -> bool {
        const uint32_t hb = hg & 1;
        if (first && !wait_bar(S.bar(B_O_FREE), (hu & 1) ^ 1, false, abort, p.status, peer_abort)) return false;
        if (!wait_bar(S.bar(B_P_FULL + hb), (hg >> 1) & 1, false, abort, p.status, peer_abort)) return false;
        MLA_TRACE_EV(hg, 22);
        ptx::tc_fence_after();
        const uint32_t kt = S.base + SK0 + hb * SK_STRIDE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = ptx::smem_desc(kt + kk * 2048, 8192, 1024, ptx::SW_128B);
          ptx::mma_ts(tbase + T_O, tbase + T_S + 64 * hb + 8 * kk, bd, IDESC_PV, (first && kk == 0) ? 0u : 1u);
        }
        ptx::mma_commit(S.bar(B_O_DONE + hb));
        ptx::mma_commit(S.bar(B_K_EMPTY + hb));
        MLA_TRACE_EV(hg, 23);
        return true;
      };
      while (wk.next(u)) {
        MLA_WAIT(S.bar(B_Q_FULL), uu & 1, false);
        ptx::tc_fence_after();
        for (int j = u.tb; j < u.te; ++j, ++g) {
          const uint32_t kb = g & 1;
          MLA_WAIT(S.bar(B_K_FULL + kb), (g >> 1) & 1, false);
          MLA_TRACE_EV(g, 20);
          ptx::tc_fence_after();
          const uint32_t kt = S.base + SK0 + kb * SK_STRIDE;
          const uint32_t dS = tbase + T_S + 64 * kb;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            const uint64_t ad = ptx::smem_desc(S.base + SQ_LAT + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, ptx::SW_128B);
            const uint64_t bd = ptx::smem_desc(kt + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, ptx::SW_128B);
            ptx::mma_ss(dS, ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t ad = ptx::smem_desc(S.base + SQ_ROPE + ks * 32, 16, 512, ptx::SW_64B);
            const uint64_t bd = ptx::smem_desc(kt + SK_ROPE + ks * 32, 16, 512, ptx::SW_64B);
            ptx::mma_ss(dS, ad, bd, IDESC_QK, 1u);
          }
          ptx::mma_commit(S.bar(B_S_FULL + kb));
          MLA_TRACE_EV(g, 21);
          if (j == u.te - 1) ptx::mma_commit(S.bar(B_Q_FREE));
          if (have_prev && !issue_pv(prev_g, prev_first, prev_u)) goto role_done;
          have_prev = true;
          prev_g = g;
          prev_first = (j == u.tb);
          prev_u = uu;
        }
        ++uu;
      }
      if (have_prev && !issue_pv(prev_g, prev_first, prev_u)) goto role_done;
    }
  }
role_done:
#undef MLA_WAIT
#undef MLA_WAIT_WARP
  // every tcgen05 op issued by the MMA thread has finished before TMEM is released
  if (warp == 9 && lane == 0) {
    ptx::mma_commit(S.bar(B_DRAIN));
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(S.bar(B_DRAIN), 0) && ptx::globaltimer() - t0 < WAIT_LIMIT_NS) {}
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // no DSMEM traffic targets a CTA that has exited
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, TMEM_COLS);
  }
}

// =============================================================================================
// plan kernel: per-item visible keys and tile prefix, per-cluster first item (1 CTA)
// =============================================================================================
constexpr int PLAN_THREADS = 1024;

__global__ void __launch_bounds__(PLAN_THREADS)
mla_plan_kernel(const uint32_t* __restrict__ cache_lengths, int B, int T, int G, uint32_t max_cache_length,
                int NC, int32_t* item_start, int32_t* item_nvis, int32_t* cluster_first, int32_t* hdr,
                unsigned int* status) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int items = B * T * G;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  if (t == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < items; base += PLAN_THREADS) {
    const int it = base + t;
    int tiles = 0;
    if (it < items) {
      const int b = it / (T * G);
      const int i = (it / G) % T;
      uint32_t L = cache_lengths[b];
      if (L > max_cache_length) {
        L = max_cache_length;
        atomicOr(status, STATUS_BOUNDS);
      }
      const int nvis = static_cast<int>(L) + i + 1;
      item_nvis[it] = nvis;
      tiles = (nvis + BN - 1) / BN;
    }
    int v = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[w] = v;
    __syncthreads();
    if (w == 0) {
      int s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += n;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int excl = carry + (w ? warp_sums[w - 1] : 0) + v - tiles;
    if (it < items) item_start[it] = excl;
    __syncthreads();
    if (t == 0) carry += warp_sums[31];
    __syncthreads();
  }
  const int total = carry;
  const int tpc = max(1, (total + NC - 1) / NC);
  if (t == 0) {
    item_start[items] = total;
    hdr[0] = tpc;
    hdr[1] = total;
  }
  __syncthreads();
  for (int kk = t; kk < NC; kk += PLAN_THREADS) {
    const int t0 = kk * tpc;
    int first = items;
    if (t0 < total) {
      int lo = 0, hi = items - 1;        // largest it with item_start[it] <= t0
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (item_start[mid] <= t0) lo = mid; else hi = mid - 1;
      }
      first = lo;
    }
    cluster_first[kk] = first;
  }
}

// =============================================================================================
// split-KV combine: lse = log sum_s e^{lse_s}; out = sum_s e^{lse_s - lse} out_s  (one warp per head)
// =============================================================================================
constexpr int COMBINE_HEADS = 8;

__global__ void __launch_bounds__(32 * COMBINE_HEADS)
mla_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int per_item = MROWS / COMBINE_HEADS;
  const int it = blockIdx.x / per_item;
  const int hc = blockIdx.x % per_item;
  if (it >= p.items) return;
  const int tpc = p.hdr[0];
  const int s = p.item_start[it], e = p.item_start[it + 1];
  const int k0 = s / tpc, k1 = (e - 1) / tpc;
  if (k0 == k1) return;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = hc * COMBINE_HEADS + w;
  const int g = it % p.G, i = (it / p.G) % p.T, b = it / (p.G * p.T);
  const int head = g * MROWS + h;
  if (head >= p.H) return;
  float mx = -INFINITY;
  for (int kk = k0; kk <= k1; ++kk) {
    const int slot = 2 * kk + (max(s, kk * tpc) == kk * tpc ? 0 : 1);
    mx = fmaxf(mx, p.part_lse[slot * MROWS + h]);
  }
  float4 acc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  float tot = 0.f;
  for (int kk = k0; kk <= k1; ++kk) {
    const int slot = 2 * kk + (max(s, kk * tpc) == kk * tpc ? 0 : 1);
    const float wgt = __expf(p.part_lse[slot * MROWS + h] - mx);
    tot += wgt;
    const float4* src = reinterpret_cast<const float4*>(p.part_o + (static_cast<size_t>(slot) * MROWS + h) * V_DIM);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = src[j * 32 + lane];
      acc[j].x += wgt * v.x;
      acc[j].y += wgt * v.y;
      acc[j].z += wgt * v.z;
      acc[j].w += wgt * v.w;
    }
  }
  const float inv = 1.f / tot;
  uint16_t* dst = p.out + ((static_cast<size_t>(b) * p.T + i) * p.H + head) * V_DIM;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint2 o;
    o.x = ptx::pack_bf16x2(acc[j].x * inv, acc[j].y * inv);
    o.y = ptx::pack_bf16x2(acc[j].z * inv, acc[j].w * inv);
    reinterpret_cast<uint2*>(dst)[j * 32 + lane] = o;
  }
  if (lane == 0 && p.lse) p.lse[(static_cast<size_t>(b) * p.T + i) * p.H + head] = mx + __logf(tot);
}

// =============================================================================================
// gather + dequant kernel (steps A and C alone): one CTA per (request, tile, dim half)
// =============================================================================================
constexpr int DQ_THREADS = 160;
constexpr uint32_t DQ_SK = 0;                    // bf16 tile (SK_STRIDE bytes)
constexpr uint32_t DQ_SF = SK_STRIDE;            // FP8 stage (SF_STRIDE bytes), 1024-aligned
constexpr uint32_t DQ_BAR = DQ_SF + SF_STRIDE;
constexpr uint32_t DQ_SMEM_ALLOC = DQ_BAR + 64 + 1024;

__global__ void __launch_bounds__(DQ_THREADS)
mla_dequant_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tm_lat,
                   const __grid_constant__ CUtensorMap tm_rope, const uint32_t* cache_lengths, int max_keys,
                   int tiles_per_req, uint16_t* out_k) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = ptx::smem_u32(smem);
  const int b = blockIdx.x / tiles_per_req;
  const int j = blockIdx.x % tiles_per_req;
  const int c = blockIdx.y;
  const int n = min(static_cast<int>(min(cache_lengths[b], 0x3FFFFFFFu)) + p.T, max_keys);
  if (j * BN >= n || b >= p.B) return;
  const int nv = min(BN, n - j * BN);
  const uint32_t full = base + DQ_BAR;
  if (threadIdx.x == 0) {
    ptx::mbar_init(full, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 128) produce_tile(p, &tm_lat, &tm_rope, c, b, j * BN, nv, base + DQ_SF, full);
  // bounded wait for the stage
  {
    const uint64_t t0 = ptx::globaltimer();
    bool ok = false;
    while (!(ok = ptx::mbar_try_wait(full, 0)) && ptx::globaltimer() - t0 < WAIT_LIMIT_NS) {}
    if (!ok) {
      if (threadIdx.x == 0) raise_status(p.status, STATUS_TIMEOUT);
      return;
    }
  }
  if (threadIdx.x < 128) convert_tile(threadIdx.x, base + DQ_SF, base + DQ_SK, nv);
  __syncthreads();
  // un-swizzle the tile back to row-major [row][576] bf16
  for (int id = threadIdx.x; id < BN * 36; id += DQ_THREADS) {
    const int row = id / 36, cc = id - row * 36;
    if (row >= nv) continue;
    uint32_t src;
    int col;
    if (cc < 32) {
      src = base + DQ_SK + (cc >> 3) * 8192 + sw128_off(row, cc & 7);
      col = 256 * c + cc * 8;
    } else {
      src = base + DQ_SK + SK_ROPE + sw64_off(row, cc - 32);
      col = 512 + 32 * c + (cc - 32) * 8;
    }
    const uint4 v = ptx::ld_shared_v4(src);
    uint16_t* dst = out_k + (static_cast<size_t>(b) * max_keys + j * BN + row) * HEAD_DIM + col;
    *reinterpret_cast<uint4*>(dst) = v;
  }
}

}  // namespace mla
