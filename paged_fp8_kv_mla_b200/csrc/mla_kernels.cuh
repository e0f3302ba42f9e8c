// Device code of the paged FP8-KV MLA decode for sm_100a.
//
// Work decomposition.  An "item" is one (request b, query token i, group of 128 query heads g).
// Item keys are tiled in BN = 64-key tiles; all items' tiles are laid end to end and cut into
// equal contiguous ranges, one per 2-CTA cluster.  A cluster walks the pieces ("units") of the
// items in its range.  An item cut by a range boundary is "split": each piece writes a normalised
// fp32 partial and its LSE, and the combine kernel merges them.
//
// The two CTAs of a cluster form one tcgen05 CTA pair (cta_group::2).  Pair MMAs have M = 128:
// CTA c supplies rows 64c..64c+63 of A and half of B along N, and receives rows 64c..64c+63 of D
// in its tensor memory (row r's first N/2 columns in TMEM lane r, the other N/2 in lane r + 64).
//   Q.K^T : A = Q (CTA c holds heads 64c..64c+63, all 576 dims), B = the 64 keys of a tile
//           (CTA c holds keys 32c..32c+31, all 576 dims).  Each CTA gets complete score rows for
//           its 64 heads, so the softmax needs no cross-CTA exchange.
//   P.V   : two MMAs of N = 256 (V dims 0..255 and 256..511).  A = P (CTA c's 64 heads, 64 keys);
//           B = V split along N: CTA c holds, for all 64 keys of the tile, the V dims
//           D_c = [128c, 128c+128) u [256+128c, 256+128c+128).  Its own 32 keys' D_c dims come from
//           the same conversion as its K half; it dequantises the other CTA's 32 keys' D_c dims
//           itself (256 of their 576 bytes), so no converted data crosses between SMs.
// Every KV byte is read from HBM once (the other CTA's partial reads hit L2).
//
// The FP8 pages reach shared memory through a two-stage ring ("KVLoad2CvtProducer", which stages
// FP8 tiles in shared memory for converter warps behind a producer): per tile, CTA c's producer
// bulk-copies its own 32 keys' rows (one contiguous 18 KB run per page) and the per-token scales of
// all 64 keys into a stage, with a full / empty mbarrier pair per stage.
//
// Buffering: K halves are double buffered (K of tile g+1 is converted while Q.K^T(g) runs), the V
// operand and P are single buffered (V(g) and P(g) are written once P.V(g-1) has finished, while
// the tensor pipe runs Q.K^T(g+1)).
//
// Warp roles per CTA (640 threads):
//   warps 0-11  converter, three groups of four warps (one warp of each group per scheduler).  In
//               step g group q dequantises atom columns 3q..3q+2 (192 dims) of the CTA's own 32
//               keys of tile g from the ring into K half buffer g % 2 (free once Q.K^T(g-2) has
//               finished), then writes its share of tile g-1's V operand (once P.V(g-2) has
//               finished).  The other CTA's keys' D_c bytes are loaded from global memory (they are
//               in L2: the other CTA's producer brought them) a step ahead.
//   warps 12-15 softmax: online softmax of the CTA's 64 heads (two lanes per head row), P -> SMEM,
//               lazy O rescale, epilogue
//   warp 16     Q.K^T issuer (CTA 0 of the pair; one elected lane issues) and TMEM owner (pair
//               allocation in both CTAs)
//   warp 17     P.V issuer (CTA 0)
//   warp 18     Q loader: one TMA tile load of the CTA's 64 heads x 576 dims per unit
//   warp 19     FP8 producer: page-table lookup and bulk copies of the ring (one elected lane)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"

namespace mla {

constexpr int BN = 64;          // keys per tile (both CTAs)
constexpr int HALF_BN = 32;     // keys per CTA in the Q.K^T B operand
constexpr int HEAD_DIM = 576;
constexpr int V_DIM = 512;
constexpr int MROWS = 128;      // query heads per item (pair MMA M)
constexpr int HPC = 64;         // query heads per CTA
constexpr int CONV_WARPS = 12;
constexpr int CONV_THREADS = 32 * CONV_WARPS;
constexpr int CONV_GROUP = 128;  // threads per converter group (three groups, 3 atom columns each)
constexpr int SM_WARP0 = 12;    // first softmax warp (warps 12..15 reach TMEM lane quadrants 0..3)
constexpr int QK_WARP = 16;     // Q.K^T issuer (CTA 0), TMEM owner (both CTAs)
constexpr int PV_WARP = 17;     // P.V issuer (CTA 0)
constexpr int Q_WARP = 18;      // Q tile loader
constexpr int LOAD_WARP = 19;   // FP8 producer
constexpr int NUM_THREADS = 640;
static_assert(SM_WARP0 % 4 == 0, "softmax warps must start a warpgroup (TMEM lane quadrants)");

// ---- shared memory map (offsets from a 1024-byte aligned base); all bf16 operands K-major
//      SWIZZLE_128B, one "atom column" = 64 bf16 dims x rows at 128 B, 8-row groups 1024 B apart
constexpr uint32_t SQ = 0;                       // Q: 9 atom columns x (64 rows x 128 B)
constexpr uint32_t SQ_ATOM = 8192;
constexpr uint32_t SK0 = 9 * SQ_ATOM;            // K half (2 buffers): 9 atom columns x (32 rows x 128 B)
constexpr uint32_t SK_ATOM = 4096;
constexpr uint32_t SK_STRIDE = 9 * SK_ATOM;
constexpr uint32_t SV = SK0 + 2 * SK_STRIDE;     // V operand (1 buffer): 4 atom columns x (64 rows x 128 B)
constexpr uint32_t SV_ATOM = 8192;
constexpr uint32_t SV_BYTES = 4 * SV_ATOM;
constexpr uint32_t SP = SV + SV_BYTES;           // P (1 buffer): 64 rows x 128 B; epilogue staging
constexpr uint32_t SP_BYTES = 8192;
constexpr uint32_t SRING = SP + SP_BYTES;        // FP8 ring (2 stages): 32 rows x 576 B, 32 own + 32 other scales
constexpr uint32_t RING_ROWS = HALF_BN * HEAD_DIM;
constexpr uint32_t RING_OSC = RING_ROWS + HALF_BN * 4;   // the other CTA's keys' scales
constexpr uint32_t RING_STAGE = RING_OSC + HALF_BN * 4;
constexpr uint32_t SRED = SRING + 2 * RING_STAGE;   // row-max exchange [2][128] f32, row-sum exchange [128] f32
constexpr uint32_t SBAR = SRED + 1536;
constexpr uint32_t SMEM_USED = SBAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;   // slack for aligning the base
static_assert(SMEM_ALLOC <= 232448, "shared memory map exceeds 227 KB");
static_assert(RING_STAGE % 16 == 0 && SRING % 16 == 0, "bulk copies need 16-byte aligned stages");
// Scale-folding mode only: the per-token scales of the last eight tiles ([8][64] f32), handed from
// the converter to the softmax warps.  It sits after SMEM_USED, inside the alignment slack, with
// the allocation at the 227 KB limit; the kernel checks that the base needed at most
// SMEM_FOLD_MAX_PAD bytes of alignment (it needs none when the runtime places dynamic shared
// memory on a 1 KB boundary) and reports STATUS_LAYOUT otherwise.
constexpr uint32_t SSC = SMEM_USED;
constexpr uint32_t SSC_STRIDE = 64 * 4;
constexpr uint32_t SSC_SLOTS = 8;
// FP8 P.V mode only: per scale slot, the largest scale of the tile seen by each of the four
// converter warps that write SSC ([8][4] f32).
constexpr uint32_t SSMAX = SSC + SSC_SLOTS * SSC_STRIDE;
constexpr uint32_t SMEM_ALLOC_FOLD = 232448;
constexpr uint32_t SMEM_FOLD_MAX_PAD = SMEM_ALLOC_FOLD - SSMAX - SSC_SLOTS * 16;
static_assert(SMEM_ALLOC_FOLD >= SSMAX + SSC_SLOTS * 16, "fold scale array does not fit");
// FP8 P.V mode: the V operand is raw e4m3, double buffered in the bf16 V buffer's place: buffer b
// at SV + b * SV8_STRIDE holds 2 atom columns (128 dims each: D_c's two halves) of 64 key rows at
// 128 B, SWIZZLE_128B, 8-row groups 1 KB apart.  P keeps its buffer: row r holds the hi codes of the
// 64 keys in bytes 0..63 and the lo codes in bytes 64..127 (same 128-byte swizzle).
constexpr uint32_t SV8_STRIDE = 16384;
constexpr uint32_t SV8_ATOM = 8192;
static_assert(2 * SV8_STRIDE <= SV_BYTES, "FP8 V buffers do not fit the V buffer");
// e4m3 P.V mode: the largest folded scale s_max * 2^sigma is at most 448 / 4, and the softmax keeps
// its reference maximum within 2 (log2 units) of the running maximum, so p <= 4 and every weight
// p * s * 2^sigma <= 448.
constexpr float FP8_PV_LAZY_LOG2 = 2.f;
// Block-scale mode with g <= 9 only (SCALE_BLOCKR): per ring stage the g scales of each of the 32
// own keys (32 x g fp32, row r at 4 g r), after SMEM_USED like the scale-folding arrays (which this
// mode does not use), inside the larger allocation.
constexpr uint32_t SBSC = SMEM_USED;
constexpr int BSC_MAX_G = 9;
constexpr uint32_t BSC_STRIDE = HALF_BN * BSC_MAX_G * 4;
static_assert(SBSC + 2 * BSC_STRIDE + 1023 <= SMEM_ALLOC_FOLD, "block-scale stages do not fit");

// How the per-token scale enters the computation.
enum ScaleMode : int {
  SCALE_TOKEN = 0,   // K, V = bf16_rn(f32_rn(e4m3 * s_t)), one scale per token
  SCALE_BLOCK = 1,   // the same with g scales per token, each over 576 / g contiguous dims
  SCALE_FOLD = 2,    // K, V = exact e4m3 values; s_t scales score column t and weight column t
  SCALE_FP8PV = 3,   // K as SCALE_TOKEN; P.V in e4m3: V = raw e4m3 bytes, s_t (and 2^sigma) carried by
                     // the weights, each weight split into two e4m3 terms
  SCALE_BLOCKR = 4   // SCALE_BLOCK for g <= 9: the own keys' block scales come through the ring (SBSC)
};

enum Bar : uint32_t {
  B_K_FULL = 0,       // [2] CTA 0: 24 warp arrivals (12 converter warps of each CTA): K half converted
  B_V_FULL = 2,       // [2] CTA 0: 24 warp arrivals: V operand converted (alternates by tile parity)
  B_PV_DONE = 4,      // [2] both CTAs: pair commit after P.V of a tile (the V and P buffers are free)
  B_S_FULL = 6,       // [2] both CTAs: pair commit after Q.K^T of a tile (S ready, its K buffer free)
  B_S_FREE = 8,       // [2] CTA 0: 8 warp arrivals (4 softmax warps of each CTA hold S in registers)
  B_P_FULL = 10,      // [2] CTA 0: 8 warp arrivals (alternates by tile parity)
  B_Q_FULL = 12,      // CTA 0: 2 arrivals (the Q loader of each CTA)
  B_Q_FREE = 13,      // both CTAs: pair commit after the last Q.K^T of a unit
  B_Q_LOCAL = 14,     // both CTAs: transaction barrier of this CTA's Q tile load
  B_O_FREE = 15,      // CTA 0: 8 warp arrivals after each CTA's epilogue
  B_DRAIN = 16,       // CTA 0: one commit from each issuer at exit
  B_RED = 17,         // [2][2] softmax warps of this CTA, by tile parity and warp pair (warps q and q + 2
                      // hold the two halves of the same head rows): row-max exchange (2 warp arrivals)
  B_REDL = 21,        // [2] by warp pair: row-sum exchange at a unit's end (2 warp arrivals)
  B_EXIT = 23,        // both CTAs: the peer has finished (1 remote arrival)
  B_RING_FULL = 24,   // [2] this CTA: the producer's expect_tx arrival + the stage's bulk-copy bytes
  B_RING_EMPTY = 26,  // [2] this CTA: 12 converter-warp arrivals, the stage has been read
  B_SC_FULL = 28,     // [8] scale-folding mode: 12 converter-warp arrivals, a tile's scales are in SSC
  NUM_BARS = 36
};
static_assert(8 * NUM_BARS <= 480, "barrier block overlaps the scalars after it");
constexpr uint32_t S_MASK = SBAR + 480;      // [2][2] u32: per ring stage, own rows copied, other scales copied
constexpr uint32_t S_TMEM_BASE = SBAR + 496;
constexpr uint32_t S_ABORT = SBAR + 500;

// TMEM columns (pair layout)
constexpr uint32_t T_O = 0;                      // P.V halves: cols 0..127 (dims 0..255), 128..255 (256..511)
constexpr uint32_t T_S = 256;                    // + 32 * buffer
constexpr uint32_t T_Q = 320;                    // Q dims 0..383 (atom columns 0..5), 2 bf16 per column,
                                                 // head row r in lanes r and r + 64
constexpr int Q_TMEM_ATOMS = 6;
constexpr uint32_t TMEM_COLS = 512;
static_assert(T_Q + 32 * Q_TMEM_ATOMS <= TMEM_COLS, "tensor memory map overflows");

constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(128, BN, false, false);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, 256, false, true);
constexpr uint32_t IDESC_PV8 = ptx::idesc_e4m3_f32(128, 256, false, true);

constexpr unsigned STATUS_BOUNDS = 1u;
constexpr unsigned STATUS_TIMEOUT = 2u;
constexpr unsigned STATUS_LAYOUT = 4u;   // the shared-memory base was not aligned as the fold mode needs
constexpr uint64_t DEFAULT_WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait unless the caller sets another

// Test hook (DecodeParams::inject): the Q loader of CTA 1 of cluster 0 withholds its arrival on the
// first unit's Q_FULL barrier, so the Q.K^T issuer's bounded wait runs out.
constexpr int INJECT_NONE = 0;
constexpr int INJECT_SKIP_Q_ARRIVAL = 1;

// Optional per-stage timestamps (build with -DMLA_TRACE): cluster 0 writes %clock64 values to
// trace[(cta * TRACE_TILES + tile) * TRACE_EVENTS + event] for its first TRACE_TILES tiles.
constexpr int TRACE_TILES = 64;
constexpr int TRACE_EVENTS = 64;   // 0..31 role stages, 32..43 K done per converter warp, 44..55 V done

// Unsigned 32-bit division by a divisor fixed for the launch, as a multiply-high and two shifts
// (Granlund and Montgomery, "Division by invariant integers using multiplication", 1994, Fig. 4.1):
// with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
//   t = mulhi(m, n),  q = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0)
// is exact for every 32-bit n.  The host fills the fields (make_fastdiv in the library).
struct FastDiv {
  uint32_t d, m, s1, s2;
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    const uint32_t t = __umulhi(n, m);
    return (t + ((n - t) >> s1)) >> s2;
  }
  __device__ __forceinline__ uint32_t mod(uint32_t n) const { return n - div(n) * d; }
};

struct DecodeParams {
  CUtensorMap tmap_q;              // q as [B*T][H][576] bf16, box 64 dims x 64 heads, SWIZZLE_128B
  unsigned long long* trace;       // null unless tracing
  const uint16_t* q;               // bf16 bits [B, T, H, 576]
  const uint8_t* blocks;           // e4m3 [NB, KVD, NL, P, 1, 576]
  const float* scales;             // fp32 [NSB, KVD, NL, P, 1, SG]
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
  unsigned long long wait_limit_ns;   // bound of every mbarrier wait in the decode kernel
  int inject;                      // INJECT_NONE, or a test hook that withholds one arrival
  int B, T, H, G, P, KVD, NL, layer, NB, NSB, max_pages, items, NC;
  FastDiv divP, divG, divT;        // by the page size, the head-group count and the query length
  int SG;                          // scales per token (head_dim_granularity): 1, or g with 576 / g % 16 == 0
  FastDiv divCPB;                  // 16-byte chunks per scale block (36 / g)
  float scale_log2;                // softmax_scale * log2(e)
};

struct Unit {
  int item, b, i, g, nvis;
  int tb, te;       // tile range within the item
  int slot;         // partial slot, -1 = write out directly
};

// Walks the units of cluster `k`: the pieces of items inside tile range [R0, R1).  The kernel
// parameters are passed to each call rather than stored (fewer live registers in the loops).
struct UnitWalker {
  int k, R0, R1, it;
  __device__ UnitWalker(const DecodeParams& p, int k_) : k(k_) {
    const int tpc = p.hdr[0], total = p.hdr[1];
    R0 = k * tpc;
    R1 = min(total, R0 + tpc);
    it = p.cluster_first[k];
  }
  __device__ bool next(const DecodeParams& p, Unit& u) {
    if (R0 >= R1 || it >= p.items) return false;
    const int s = p.item_start[it], e = p.item_start[it + 1];
    const int a = max(s, R0), z = min(e, R1);
    if (a >= z) return false;
    u.item = it;
    const uint32_t bi = p.divG.div(it);       // it = (b * T + i) * G + g
    u.g = it - static_cast<int>(bi) * p.G;
    u.b = static_cast<int>(p.divT.div(bi));
    u.i = static_cast<int>(bi) - u.b * p.T;
    u.nvis = p.item_nvis[it];
    u.tb = a - s;
    u.te = z - s;
    const bool split = (s < R0) || (e > R1);
    u.slot = split ? (2 * k + (a == R0 ? 0 : 1)) : -1;
    ++it;
    return true;
  }
};

__device__ unsigned int g_status_word;   // sticky device status (bit 0 bounds, bit 1 timeout)

__device__ __forceinline__ void raise_status(unsigned int* status, unsigned bits) {
  atomicOr(status ? status : &g_status_word, bits);
}

#ifdef MLA_TRACE
#define MLA_TRACE_EV(tile, ev)                                                                        \
  do {                                                                                                \
    if (p.trace && k == 0 && (tile) < static_cast<uint32_t>(TRACE_TILES))                            \
      p.trace[(c * TRACE_TILES + (tile)) * TRACE_EVENTS + (ev)] = clock64();                         \
  } while (0)
#else
#define MLA_TRACE_EV(tile, ev) do {} while (0)
#endif
// Trace builds also record, per CTA, %globaltimer at entry, after setup and at exit, at
// trace[2 * TRACE_TILES * TRACE_EVENTS + 4 * blockIdx.x + {0, 1, 2}].
#ifdef MLA_TRACE
// Trace builds: %globaltimer marks of one decode call: [0] plan end, [1] first decode CTA entry,
// [2] last decode CTA exit, [3] first combine CTA past its grid-dependency wait, [4] last combine
// warp done, [5] first combine CTA entry.
__device__ unsigned long long g_trace_marks[8];
#define MLA_MARK_MIN(i) atomicMin(&g_trace_marks[i], static_cast<unsigned long long>(ptx::globaltimer()))
#define MLA_MARK_MAX(i) atomicMax(&g_trace_marks[i], static_cast<unsigned long long>(ptx::globaltimer()))
#else
#define MLA_MARK_MIN(i) do {} while (0)
#define MLA_MARK_MAX(i) do {} while (0)
#endif
#ifdef MLA_TRACE
#define MLA_TRACE_CTA(slot)                                                                           \
  do {                                                                                                \
    if (p.trace && threadIdx.x == 0)                                                                  \
      p.trace[2 * TRACE_TILES * TRACE_EVENTS + 4 * blockIdx.x + (slot)] = ptx::globaltimer();         \
  } while (0)
#else
#define MLA_TRACE_CTA(slot) do {} while (0)
#endif

// Bounded wait on an mbarrier phase (CTA-scope acquire; barriers arrived on by this CTA's threads,
// by the peer CTA's threads through remote arrives, by tcgen05 commits or by bulk-copy bytes).
// Returns false when the wait gives up or another role already gave up; the first to give up
// marks the CTA, its peer and the status word.  The loop is kept small (it is inlined at every
// wait) and the give-up path is out of line.
__device__ __noinline__ bool wait_gave_up(volatile uint32_t* abort, unsigned int* status, uint32_t peer_abort) {
  if (!*abort) {
    *abort = 1u;
    if (peer_abort) ptx::st_cluster_u32(peer_abort, 1u);
    raise_status(status, STATUS_TIMEOUT);
  }
  return false;
}

__device__ __forceinline__ bool wait_bar(uint32_t addr, uint32_t parity, volatile uint32_t* abort,
                                         unsigned int* status, uint32_t peer_abort, uint64_t limit) {
  if (ptx::mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait_sleep(addr, parity, 20000u)) {
    if (*abort) return false;
    if (ptx::globaltimer() - t0 > limit) return wait_gave_up(abort, status, peer_abort);
  }
  return true;
}

// The same bound, polling instead of suspending in try_wait: the MMA issuers and the converter's
// K-buffer wait use it because a suspended thread resumes hundreds of cycles after the phase
// completes, and those waits sit on the critical path of every tile.
__device__ __forceinline__ bool poll_bar(uint32_t addr, uint32_t parity, volatile uint32_t* abort,
                                         unsigned int* status, uint32_t peer_abort, uint64_t limit) {
  if (ptx::mbar_test_wait(addr, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_test_wait(addr, parity)) {
    __nanosleep(32);
    if (*abort) return false;
    if (ptx::globaltimer() - t0 > limit) return wait_gave_up(abort, status, peer_abort);
  }
  return true;
}

// Time-bounded wait that ignores the abort flag: for the completion of this CTA's own bulk copies
// and TMA loads before it exits (they land whatever the other roles did).
__device__ __forceinline__ void drain_bar(uint32_t addr, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(addr, parity) && ptx::globaltimer() - t0 < limit) {}
}

// ---------------------------------------------------------------------------------------------
// Dequantisation of 16 e4m3 bytes of one row with the row's scale -> 16 bf16 (8 packed words):
// bf16_rn(f32_rn(e4m3 * s)).  e4m3 -> f16 -> f32 is exact; the multiply rounds to nearest in fp32;
// the pack rounds to nearest-even bf16.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void dequant16(uint4 raw, float s, uint32_t (&w)[8]) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
  const float2 ss = make_float2(s, s);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t h0 = ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] & 0xFFFFu));
    const uint32_t h1 = ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] >> 16));
    // packed fp32 multiply (two round-to-nearest products per instruction)
    const float2 p0 = __fmul2_rn(make_float2(ptx::f16_lo_to_f32(h0), ptx::f16_hi_to_f32(h0)), ss);
    const float2 p1 = __fmul2_rn(make_float2(ptx::f16_lo_to_f32(h1), ptx::f16_hi_to_f32(h1)), ss);
    w[2 * k] = ptx::pack_bf16x2(p0.x, p0.y);
    w[2 * k + 1] = ptx::pack_bf16x2(p1.x, p1.y);
  }
}

// Scale-folding mode: 16 e4m3 bytes -> 16 bf16 values, exactly (no scale).  e4m3 -> f16 is exact
// (every e4m3 value is a normal f16 or zero, f16 exponent field 6..23 for nonzero values, low 3
// mantissa bits zero).  Shifting the f16 magnitude bits right by 3 lines its exponent and top 7
// mantissa bits up with the bf16 fields, which reads as the same value times 2^-112 (a normal bf16
// for nonzero values, zero for zero); the sign bit is put back in place and one packed bf16
// multiply by 2^112 (exact: a power of two, result exponent field 118..135) restores the value.
__device__ __forceinline__ uint32_t f16x2_to_bf16x2_e4m3(uint32_t h) {
  const uint32_t mag = (h >> 3) & 0x0FFF0FFFu;
  return ptx::mul_bf16x2(mag | (h & 0x80008000u), 0x77807780u);   // 0x7780 = bf16 2^112
}

__device__ __forceinline__ void exact16(uint4 raw, uint32_t (&w)[8]) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    w[2 * k] = f16x2_to_bf16x2_e4m3(ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] & 0xFFFFu)));
    w[2 * k + 1] = f16x2_to_bf16x2_e4m3(ptx::e4m3x2_to_f16x2(static_cast<uint16_t>(in[k] >> 16)));
  }
}

template <bool FOLD>
__device__ __forceinline__ void convert16(bool ok, uint4 raw, float s, uint32_t (&w)[8]) {
  if (ok) {
    if (FOLD) {
      exact16(raw, w);
    } else {
      dequant16(raw, s, w);
    }
  } else {
#pragma unroll
    for (int x = 0; x < 8; ++x) w[x] = 0u;
  }
}

// Byte offset of 16-byte unit `u` (0..7) of row `r` in a K-major SWIZZLE_128B atom column whose
// 8-row groups are 1024 B apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int u) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4);
}

// One 16-dim chunk (32 bytes of bf16) at chunk position cq (0..3) of an atom column's row.
__device__ __forceinline__ void st_chunk(uint32_t atom_base, int row, int cq, const uint32_t (&w)[8]) {
  ptx::st_shared_v4(atom_base + sw128_off(row, 2 * cq), w[0], w[1], w[2], w[3]);
  ptx::st_shared_v4(atom_base + sw128_off(row, 2 * cq + 1), w[4], w[5], w[6], w[7]);
}

// Converter thread layout.  Thread t (0..383) is in group q = t / 128; thread tau = t % 128 of a
// group owns key row conv_row(tau) (0..31) and chunk position conv_cq(tau) (0..3) of each 64-dim
// atom column the group handles.  The 8 threads of one 16-byte shared-memory phase cover the 4
// chunk positions of rows r and r ^ 5 (r even), which differ in bits 0 and 2.  So their 32-byte
// bf16 stores land on 8 different 16-byte positions of the 128-byte swizzle row (even rows on even
// positions, odd rows on odd ones); their 16-byte e4m3 stores (4 adjacent positions per row) land
// in opposite halves of the swizzle row; and their 16-byte reads of the FP8 ring (576-byte rows:
// rows an odd number apart start 16 banks apart) hit 8 distinct bank quads.
__device__ __forceinline__ int conv_row(int tau) { return ((tau >> 3) << 1) ^ (((tau >> 2) & 1) * 5); }
__device__ __forceinline__ int conv_cq(int tau) { return tau & 3; }

// V atom column va (0..3) of CTA c's V operand holds the 64 dims of absolute atom column
// v_atom(va, c) (D_c = atom columns 2c, 2c+1, 4+2c, 5+2c); a K atom column a belongs to D_c when
// it is one of these, at V atom column k_to_v(a, c).
__device__ __forceinline__ int v_atom(int va, int c) { return va < 2 ? 2 * c + va : 4 + 2 * c + (va - 2); }
__device__ __forceinline__ bool k_in_dc(int a, int c) { return a < 8 && ((a >> 1) == c || (a >> 1) == 2 + c); }
__device__ __forceinline__ int k_to_v(int a, int c) { return ((a >> 1) == c) ? (a & 1) : 2 + (a & 1); }

// The group that also converts V atom column 3 of the other CTA's keys (balances the work: that
// group owns no or only one of the CTA's own D_c atom columns).
__device__ __forceinline__ int extra_group(int c) { return c == 0 ? 2 : 0; }

// Request index of an item (items are ordered (b, i, g)).
__device__ __forceinline__ int item_b(const DecodeParams& p, int item) {
  return static_cast<int>(p.divT.div(p.divG.div(item)));
}

// What the converter and the producer need to know about one tile (request, query token and head
// group follow from the item index).
struct TileInfo {
  int item, nvis, j;
  bool first, valid;
};

// Produces the tile sequence of a cluster one TileInfo at a time.
struct TileStream {
  UnitWalker wk;
  int item, nvis, j, te;
  bool valid, first;
  __device__ TileStream(const DecodeParams& p, int k) : wk(p, k) { next_unit(p); }
  __device__ void next_unit(const DecodeParams& p) {
    Unit u;
    valid = wk.next(p, u);
    item = u.item;
    nvis = u.nvis;
    j = u.tb;
    te = u.te;
    first = true;
  }
  __device__ TileInfo take(const DecodeParams& p) {
    TileInfo t;
    t.item = item;
    t.nvis = nvis;
    t.j = j;
    t.first = first;
    t.valid = valid;
    if (valid) {
      ++j;
      first = false;
      if (j >= te) next_unit(p);
    }
    return t;
  }
};

// Sequential cursor over the tiles a cluster processes (unit by unit).
struct TileCursor {
  UnitWalker wk;
  Unit u;
  int j;
  bool valid, first;
  __device__ TileCursor(const DecodeParams& p, int k) : wk(p, k) {
    valid = wk.next(p, u);
    j = valid ? u.tb : 0;
    first = true;
  }
  __device__ void advance(const DecodeParams& p) {
    ++j;
    first = false;
    if (j >= u.te) {
      valid = wk.next(p, u);
      j = valid ? u.tb : 0;
      first = true;
    }
  }
};

// Page-table lookup of one key: value row and scale row (indices into blocks / scales as
// [rows][576] and [rows][SG]; both < 2^32, checked on the host).  Returns false (and sets `bad`)
// for a page past the table or an id past its pool; the key then reads as zero.
__device__ __forceinline__ bool key_rows(const DecodeParams& p, int b, int tok, uint32_t& vrow, uint32_t& srow,
                                         bool& bad) {
  const uint32_t page = p.divP.div(static_cast<uint32_t>(tok));
  const uint32_t slot = static_cast<uint32_t>(tok) - page * static_cast<uint32_t>(p.P);
  if (page >= static_cast<uint32_t>(p.max_pages)) {
    bad = true;
    return false;
  }
  const size_t e = static_cast<size_t>(b) * p.max_pages + page;
  const uint32_t blk = __ldg(p.lut + e);
  const uint32_t sblk = p.slut ? __ldg(p.slut + e) : blk;
  if (blk >= static_cast<uint32_t>(p.NB) || sblk >= static_cast<uint32_t>(p.NSB)) {
    bad = true;
    return false;
  }
  const uint32_t per_blk = static_cast<uint32_t>(p.KVD * p.NL * p.P);
  const uint32_t lay = static_cast<uint32_t>(p.layer * p.P);
  vrow = blk * per_blk + lay + slot;
  srow = sblk * per_blk + lay + slot;
  return true;
}

// ---------------------------------------------------------------------------------------------
// Producer side of one ring stage.  The keys of a half tile (n keys from token tok0 of request b)
// lie in at most two page runs (page sizes are multiples of 16 and a half tile is 32 keys; the
// second run starts on a page boundary).
// ---------------------------------------------------------------------------------------------
struct Runs {
  uint32_t v0, s0, v1, s1;     // value and scale rows of each run's first key
  int len0, len1;
  bool ok0, ok1;
};

__device__ __forceinline__ Runs half_runs(const DecodeParams& p, int b, int tok0, int n, bool& bad) {
  Runs R;
  R.v0 = R.s0 = R.v1 = R.s1 = 0;
  R.len0 = min(n, p.P - static_cast<int>(p.divP.mod(static_cast<uint32_t>(max(tok0, 0)))));
  R.ok0 = n > 0 && key_rows(p, b, tok0, R.v0, R.s0, bad);
  R.len1 = n - max(R.len0, 0);
  R.ok1 = R.len1 > 0 && key_rows(p, b, tok0 + R.len0, R.v1, R.s1, bad);
  return R;
}

__device__ __forceinline__ uint32_t run_mask(const Runs& R) {
  uint32_t m = 0;
  if (R.ok0) m |= (R.len0 >= 32 ? 0xFFFFFFFFu : ((1u << R.len0) - 1u));
  if (R.ok1) m |= ((1u << R.len1) - 1u) << R.len0;
  return m;
}

// Scale bytes of a run, rounded up to whole 16-byte units (the rounding stays inside the page:
// runs start at multiples of 16 slots and pages hold a multiple of 16).
__device__ __forceinline__ uint32_t scale_bytes(int len) { return ((static_cast<uint32_t>(len) + 3u) & ~3u) * 4u; }

// Page runs of one ring stage for tile j of request b (visible keys nvis): the CTA's own 32 keys
// and, with OTHER, the other CTA's 32 keys (whose scales only are copied).  Reads the page table;
// the producer plans a tile while the stage before it is still being read, so that the table's
// latency does not delay the copies.
struct StagePlan {
  Runs own, oth;
  bool bad;
};

template <bool OTHER>
__device__ __forceinline__ StagePlan plan_stage(const DecodeParams& p, int b, int j, int nvis, int c) {
  StagePlan sp;
  sp.bad = false;
  const int tok0 = j * BN + HALF_BN * c;
  sp.own = half_runs(p, b, tok0, max(0, min(HALF_BN, nvis - tok0)), sp.bad);
  sp.oth.ok0 = sp.oth.ok1 = false;
  sp.oth.len0 = sp.oth.len1 = 0;
  sp.oth.v0 = sp.oth.s0 = sp.oth.v1 = sp.oth.s1 = 0;
  const int tok1 = j * BN + HALF_BN * (1 - c);
  if (OTHER) sp.oth = half_runs(p, b, tok1, max(0, min(HALF_BN, nvis - tok1)), sp.bad);
  return sp;
}

// Fills one ring stage from its plan: the own keys' rows (rows [0, 32) of the stage) and, with
// per-token scales (SC), their scales at RING_ROWS; with OTHER also the other keys' scales at
// RING_OSC.  Writes the masks of copied rows and copied other-key scales to mask_addr and
// mask_addr + 4, then arrives on `full` with the byte count and issues the bulk copies.
// BSC (block-scale mode, g <= 9): also the own keys' g block scales per key, row r at
// bsc + 4 g r, one bulk copy per run rounded up to 16 bytes (the rounding stays inside the page:
// runs start at multiples of 16 slots, and a run that ends at the page's end needs none, since a
// page holds a multiple of 16 g scales).
template <bool SC, bool OTHER, bool BSC = false>
__device__ __forceinline__ void issue_planned(const DecodeParams& p, uint32_t stage, uint32_t full, uint32_t mask_addr,
                                              const StagePlan& sp, uint32_t bsc = 0) {
  const Runs& own = sp.own;
  const Runs& oth = sp.oth;
  uint32_t tx = 0;
  if (own.ok0) tx += static_cast<uint32_t>(own.len0) * HEAD_DIM + (SC ? scale_bytes(own.len0) : 0u);
  if (own.ok1) tx += static_cast<uint32_t>(own.len1) * HEAD_DIM + (SC ? scale_bytes(own.len1) : 0u);
  if (OTHER && oth.ok0) tx += scale_bytes(oth.len0);
  if (OTHER && oth.ok1) tx += scale_bytes(oth.len1);
  const uint32_t sg4 = 4u * static_cast<uint32_t>(p.SG);
  if (BSC && own.ok0) tx += (static_cast<uint32_t>(own.len0) * sg4 + 15u) & ~15u;
  if (BSC && own.ok1) tx += (static_cast<uint32_t>(own.len1) * sg4 + 15u) & ~15u;
  if (sp.bad) raise_status(p.status, STATUS_BOUNDS);
  ptx::st_shared_u32(mask_addr, run_mask(own));
  ptx::st_shared_u32(mask_addr + 4, OTHER ? run_mask(oth) : 0u);
  // The stage was last read by the converters' ordinary shared loads, which the empty-barrier
  // wait orders before this thread's later generic accesses but not before the bulk copies (async
  // proxy) that overwrite it: the proxy fence closes that write-after-read.  Without it a copy
  // issued right after the wait overwrote rows that a converter load had not yet read (seen as
  // run-to-run differences once the page-table reads no longer stood between the two).
  ptx::fence_proxy_async_smem();
  ptx::mbar_arrive_expect_tx(full, tx);
  if (own.ok0) {
    ptx::bulk_load(stage, p.blocks + static_cast<size_t>(own.v0) * HEAD_DIM, static_cast<uint32_t>(own.len0) * HEAD_DIM, full);
    if (SC) ptx::bulk_load(stage + RING_ROWS, p.scales + own.s0, scale_bytes(own.len0), full);
  }
  if (own.ok1) {
    const uint32_t r1 = static_cast<uint32_t>(own.len0);
    ptx::bulk_load(stage + r1 * HEAD_DIM, p.blocks + static_cast<size_t>(own.v1) * HEAD_DIM,
                   static_cast<uint32_t>(own.len1) * HEAD_DIM, full);
    if (SC) ptx::bulk_load(stage + RING_ROWS + 4u * r1, p.scales + own.s1, scale_bytes(own.len1), full);
  }
  if (OTHER && oth.ok0) ptx::bulk_load(stage + RING_OSC, p.scales + oth.s0, scale_bytes(oth.len0), full);
  if (OTHER && oth.ok1)
    ptx::bulk_load(stage + RING_OSC + 4u * static_cast<uint32_t>(oth.len0), p.scales + oth.s1, scale_bytes(oth.len1), full);
  if (BSC && own.ok0)
    ptx::bulk_load(bsc, p.scales + static_cast<size_t>(own.s0) * p.SG, (static_cast<uint32_t>(own.len0) * sg4 + 15u) & ~15u, full);
  if (BSC && own.ok1)
    ptx::bulk_load(bsc + static_cast<uint32_t>(own.len0) * sg4, p.scales + static_cast<size_t>(own.s1) * p.SG,
                   (static_cast<uint32_t>(own.len1) * sg4 + 15u) & ~15u, full);
}

template <bool SC, bool OTHER>
__device__ __forceinline__ void issue_stage(const DecodeParams& p, uint32_t stage, uint32_t full, uint32_t mask_addr,
                                            int b, int j, int nvis, int c) {
  issue_planned<SC, OTHER>(p, stage, full, mask_addr, plan_stage<OTHER>(p, b, j, nvis, c));
}

// Page-table entries of a converter thread's other-CTA key of one tile, read a step before the
// rows are formed from them (so that the dependent data loads do not wait on the table read).
struct OthLut {
  uint32_t blk, sblk, slot;
  bool vis, in_table;
};

__device__ __forceinline__ OthLut oth_lut_issue(const DecodeParams& p, const TileInfo& ti, int c, int r) {
  OthLut L;
  const int tok = ti.j * BN + HALF_BN * (1 - c) + r;
  const uint32_t page = p.divP.div(static_cast<uint32_t>(tok));
  L.slot = static_cast<uint32_t>(tok) - page * static_cast<uint32_t>(p.P);
  L.vis = tok < ti.nvis;
  L.in_table = page < static_cast<uint32_t>(p.max_pages);
  L.blk = L.sblk = 0;
  if (L.vis && L.in_table) {
    const size_t e = static_cast<size_t>(item_b(p, ti.item)) * p.max_pages + page;
    L.blk = __ldg(p.lut + e);
    L.sblk = p.slut ? __ldg(p.slut + e) : L.blk;
  }
  return L;
}

// Values a converter thread loads a step ahead from global memory: the other CTA's key's D_c
// chunks (V atom column = its group, and V atom column 3 for the extra group) and, in the
// block-scale mode, their scales and the scales of its own key's three K chunks.
struct Ahead {
  uint4 oth[2];
  float s_oth[2];
  float s_own[3];
  bool oth_ok, own_ok;
};

// Issues the other key's chunk loads from the table entries read by oth_lut_issue.  Returns false
// on a bad page id (that key then reads as zero).
template <bool BS>
__device__ __forceinline__ bool fetch_oth(const DecodeParams& p, const OthLut& L, int c, int grp, int cq, bool extra,
                                          Ahead& A) {
  const bool ids_ok = L.blk < static_cast<uint32_t>(p.NB) && L.sblk < static_cast<uint32_t>(p.NSB);
  const bool bad = L.vis && (!L.in_table || !ids_ok);
  A.oth_ok = L.vis && L.in_table && ids_ok;
  if (A.oth_ok) {
    const uint32_t per_blk = static_cast<uint32_t>(p.KVD * p.NL * p.P);
    const uint32_t lay = static_cast<uint32_t>(p.layer * p.P);
    const uint32_t vrow = L.blk * per_blk + lay + L.slot;
    const uint8_t* row = p.blocks + static_cast<size_t>(vrow) * HEAD_DIM;
    const int q0 = 4 * v_atom(grp, c) + cq;
    A.oth[0] = ptx::ldg_stream_v4(row + 16 * q0);
    const int q1 = 4 * v_atom(3, c) + cq;
    if (extra) A.oth[1] = ptx::ldg_stream_v4(row + 16 * q1);
    if (BS) {
      const size_t srow = static_cast<size_t>(L.sblk * per_blk + lay + L.slot) * p.SG;
      A.s_oth[0] = __ldg(p.scales + srow + p.divCPB.div(q0));
      if (extra) A.s_oth[1] = __ldg(p.scales + srow + p.divCPB.div(q1));
    }
  }
  return !bad;
}

// Block-scale mode: the scales of the thread's own key's three K chunks of one tile.
__device__ __forceinline__ bool fetch_own_scales(const DecodeParams& p, const TileInfo& ti, int c, int grp, int r,
                                                 int cq, Ahead& A) {
  bool bad = false;
  const int otok = ti.j * BN + HALF_BN * c + r;
  uint32_t ov = 0, os = 0;
  A.own_ok = otok < ti.nvis && key_rows(p, item_b(p, ti.item), otok, ov, os, bad);
  if (A.own_ok) {
#pragma unroll
    for (int m = 0; m < 3; ++m)
      A.s_own[m] = __ldg(p.scales + static_cast<size_t>(os) * p.SG + p.divCPB.div(4 * (3 * grp + m) + cq));
  }
  return !bad;
}

// K-half part of one tile for a converter thread: its three chunks of the own key's row, read from
// a ring stage (raw) and dequantised into the K half buffer at `sk`.
template <bool BS, bool FOLD>
__device__ __forceinline__ void convert_k(int grp, int r, int cq, bool ok, const uint4 (&raw)[3], float s_tok,
                                          const float (&s_blk)[3], uint32_t sk) {
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    uint32_t w[8];
    convert16<FOLD>(ok, raw[m], BS ? s_blk[m] : s_tok, w);
    st_chunk(sk + (3 * grp + m) * SK_ATOM, r, cq, w);
  }
}

// The own key's D_c chunks of a converted K half, copied into the V operand (rows 32c + r).
__device__ __forceinline__ void copy_dc_chunks(int grp, int r, int cq, int c, uint32_t sk, uint32_t sv) {
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int a = 3 * grp + m;
    if (!k_in_dc(a, c)) continue;
    const uint32_t src = sk + a * SK_ATOM, dst = sv + k_to_v(a, c) * SV_ATOM;
    const uint4 x = ptx::ld_shared_v4(src + sw128_off(r, 2 * cq));
    const uint4 y = ptx::ld_shared_v4(src + sw128_off(r, 2 * cq + 1));
    const int vr = HALF_BN * c + r;
    ptx::st_shared_v4(dst + sw128_off(vr, 2 * cq), x.x, x.y, x.z, x.w);
    ptx::st_shared_v4(dst + sw128_off(vr, 2 * cq + 1), y.x, y.y, y.z, y.w);
  }
}

// =============================================================================================
// converter role (warps 0-11); the same code in both CTAs of the pair (c = rank).
// Step g: (K) read the thread's three FP8 chunks of tile g and the tile's scales from ring stage
// g % 2 and release the stage; once Q.K^T(g-2) has finished (K half buffer g % 2 is free)
// dequantise them into it.  (V) Dequantise the other key's D_c chunks of tile g-1 (loaded during
// step g-1); once P.V(g-2) has finished (the V buffer is free) write tile g-1's V operand: those
// chunks and the own key's D_c chunks copied from K half buffer (g-1) % 2.  Then read the other
// key's chunks of tile g and the page-table entries of tile g+1.  Returns early (with the abort
// flag set by the failing wait) when a wait gives up.
// =============================================================================================
template <int MODE>
__device__ __forceinline__ void converter_role(const DecodeParams& p, int k, uint32_t base, int lane,
                                               volatile uint32_t* abort, uint32_t peer_abort, uint32_t c) {
  constexpr bool BSR = MODE == SCALE_BLOCKR;         // own block scales from the ring's side area
  constexpr bool BS = MODE == SCALE_BLOCK || BSR;
  constexpr bool FOLD = MODE == SCALE_FOLD;
  const int C = static_cast<int>(c);
  const int t = threadIdx.x;
  const int grp = t / CONV_GROUP, tau = t % CONV_GROUP;
  const int r = conv_row(tau), cq = conv_cq(tau);
  const bool extra = grp == extra_group(C);
  const uint64_t lim = p.wait_limit_ns;
#define BAR(i) (base + SBAR + 8u * (i))
#define MLA_WAIT_RET(b_, parity)                                                               \
  if (!__all_sync(0xffffffffu, wait_bar((b_), (parity), abort, p.status, peer_abort, lim))) return;
#define MLA_POLL_RET(b_, parity)                                                               \
  if (!__all_sync(0xffffffffu, poll_bar((b_), (parity), abort, p.status, peer_abort, lim))) return;
  const uint32_t k_full0 = ptx::mapa(BAR(B_K_FULL), 0), v_full0 = ptx::mapa(BAR(B_V_FULL), 0);
  TileStream ts(p, k);
  TileInfo kt = ts.take(p);
  if (!kt.valid) return;
  TileInfo nt = ts.take(p);
  OthLut L = oth_lut_issue(p, kt, C, r);
  Ahead A;                       // the other key's chunks of the tile whose V operand is written next
  A.oth_ok = false;
  A.own_ok = true;
  if (BS && !BSR && !fetch_own_scales(p, kt, C, grp, r, cq, A)) raise_status(p.status, STATUS_BOUNDS);
  float s_oth_v = 0.f;           // per-token scale of that key (from the ring)
  uint32_t g = 0;
  // Rolled loop (one copy of the step keeps the hot code small).
  while (true) {
    float s_oth_k = 0.f;
    if (kt.valid) {
      // ---------------------------------------------------------------- K half of tile g
      const uint32_t st = g & 1;
      if (t == 0) MLA_TRACE_EV(g, 1);
      MLA_WAIT_RET(BAR(B_RING_FULL + st), (g >> 1) & 1);
      if (t == 0) MLA_TRACE_EV(g, 3);
      const uint32_t stage = base + SRING + st * RING_STAGE;
      const bool own_ok = ((ptx::ld_shared_u32(base + S_MASK + 8 * st) >> r) & 1u) != 0 && A.own_ok;
      uint4 raw[3];
#pragma unroll
      for (int m = 0; m < 3; ++m) raw[m] = ptx::ld_shared_v4(stage + r * HEAD_DIM + 16 * (4 * (3 * grp + m) + cq));
      const float s_own = BS ? 0.f : ptx::ld_shared_f32(stage + RING_ROWS + 4 * r);
      if (!BS) s_oth_k = ptx::ld_shared_f32(stage + RING_OSC + 4 * r);
      if (BSR) {
        // the block scales of the thread's three chunks of its own key, from the stage's side area
        const uint32_t bsc = base + SBSC + st * BSC_STRIDE + 4u * static_cast<uint32_t>(r * p.SG);
#pragma unroll
        for (int m = 0; m < 3; ++m) A.s_own[m] = ptx::ld_shared_f32(bsc + 4u * p.divCPB.div(4 * (3 * grp + m) + cq));
      }
      if (FOLD) {
        // the tile's 64 per-token scales for the softmax (0 for keys not read).  Slot g % 8 last
        // held tile g - 8, which the softmax finished before S_FREE(g - 5), which Q.K^T(g - 3)
        // waited for before the K-buffer wait of step g - 1 passed.
        if (grp == 0 && cq == 0) {
          const uint32_t om = ptx::ld_shared_u32(base + S_MASK + 8 * st + 4);
          const uint32_t sa = base + SSC + (g % SSC_SLOTS) * SSC_STRIDE + 4 * r;
          ptx::st_shared_f32(sa + 4 * HALF_BN * C, own_ok ? s_own : 0.f);
          ptx::st_shared_f32(sa + 4 * HALF_BN * (1 - C), ((om >> r) & 1u) ? s_oth_k : 0.f);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(BAR(B_SC_FULL + (g % SSC_SLOTS)));
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(BAR(B_RING_EMPTY + st));    // the reads above are ordered before it
      // K half buffer g % 2: free once Q.K^T(g - 2) has finished
      MLA_POLL_RET(BAR(B_S_FULL + st), ((g >> 1) & 1) ^ 1);
      if (t == 0) MLA_TRACE_EV(g, 16);
      convert_k<BS, FOLD>(grp, r, cq, own_ok, raw, s_own, A.s_own, base + SK0 + st * SK_STRIDE);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(k_full0 + 8u * st);
      if (t == 0) MLA_TRACE_EV(g, 5);
      if (t == 352) MLA_TRACE_EV(g, 26);
      if (lane == 0) MLA_TRACE_EV(g, 32 + (t >> 5));
    }
    if (g > 0) {
      // ---------------------------------------------------------------- V operand of tile g - 1
      const uint32_t vt = g - 1;
      uint32_t w0[8], w1[8];
      convert16<FOLD>(A.oth_ok, A.oth[0], BS ? A.s_oth[0] : s_oth_v, w0);
      if (extra) convert16<FOLD>(A.oth_ok, A.oth[1], BS ? A.s_oth[1] : s_oth_v, w1);
      // the V buffer is free once P.V(g - 2) has finished
      if (t == 0) MLA_TRACE_EV(vt, 4);
      MLA_WAIT_RET(BAR(B_PV_DONE + (g & 1)), ((g >> 1) & 1) ^ 1);
      if (t == 0) MLA_TRACE_EV(vt, 6);
      copy_dc_chunks(grp, r, cq, C, base + SK0 + (vt & 1) * SK_STRIDE, base + SV);
      const int vrow_oth = HALF_BN * (1 - C) + r;
      st_chunk(base + SV + grp * SV_ATOM, vrow_oth, cq, w0);
      if (extra) st_chunk(base + SV + 3 * SV_ATOM, vrow_oth, cq, w1);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(v_full0 + 8u * (vt & 1));
      if (t == 0) MLA_TRACE_EV(vt, 2);
      if (t == 352) MLA_TRACE_EV(vt, 27);
      if (lane == 0) MLA_TRACE_EV(vt, 44 + (t >> 5));
    }
    if (!kt.valid) break;
    // ---------------------------------------------------------------- loads for the next step
    s_oth_v = s_oth_k;
    if (!fetch_oth<BS>(p, L, C, grp, cq, extra, A)) raise_status(p.status, STATUS_BOUNDS);
    if (nt.valid) {
      L = oth_lut_issue(p, nt, C, r);
      if (BS && !BSR && !fetch_own_scales(p, nt, C, grp, r, cq, A)) raise_status(p.status, STATUS_BOUNDS);
    }
    if (t == 0) MLA_TRACE_EV(g, 7);
    kt = nt;
    nt = ts.take(p);
    ++g;
  }
#undef MLA_POLL_RET
#undef MLA_WAIT_RET
#undef BAR
}

// Largest power of two 2^sigma with s_max * 2^sigma <= 112 = 1.75 * 2^6 (s_max a positive normal
// float), so that every folded weight p * s * 2^sigma with p <= 4 stays at or below 448:
// sigma = 133 - e - (m > 1.75), e the biased exponent and m the significand of s_max.  Clamped to
// [-120, 120].
__device__ __forceinline__ int fp8_pv_sigma(float s_max) {
  if (!(s_max > 0.f)) return 120;
  const uint32_t b = __float_as_uint(s_max);
  const int e = static_cast<int>((b >> 23) & 0xFFu);
  const int sg = 133 - e - ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return max(-120, min(120, sg));
}

__device__ __forceinline__ float exp2i(int k) { return __int_as_float((k + 127) << 23); }   // 2^k, |k| <= 126
__device__ __forceinline__ float exp2i_or_zero(int k) { return k < -126 ? 0.f : exp2i(k); }   // 2^k, k <= 126

// Two-term e4m3 split of two weights w0, w1 >= 0: hi = e4m3_rn_sat(w) from the f32 weight; the
// residual is taken in f16, lo = e4m3_rn_sat(f16_rn(w) - hi): hi is exact in f16 and the difference
// of the two f16 values is exact (they are within a few percent of each other, or hi = 0), so lo
// differs from e4m3_rn_sat(w - hi) only where the f16 rounding of w (2^-12 of w) moves the residual
// across a rounding boundary of lo; hi + lo stays within 2^-8 + 2^-12 of w in the normal range.
// Five instructions per pair (f32 residuals would take three more conversions).  w0's codes in the
// low bytes.
__device__ __forceinline__ void split2_e4m3(float w0, float w1, uint32_t& hi, uint32_t& lo) {
  const uint16_t h = ptx::e4m3x2_rn_satfinite(w0, w1);
  hi = h;
  lo = ptx::e4m3x2_rn_satfinite_f16x2(ptx::sub_f16x2(ptx::pack_f16x2(w0, w1), ptx::e4m3x2_to_f16x2(h)));
}

// 16-byte unit (0..7) of a P row that holds a softmax thread's chunk j (0..3) of its key half hh:
// bf16 P: the thread's 32 weights at units 4hh..4hh+3; e4m3 P: its 32 hi codes at units 2hh, 2hh+1
// and its 32 lo codes at units 4+2hh, 5+2hh.
template <bool F8>
__device__ __forceinline__ int p_unit(int hh, int j) {
  return F8 ? ((j >> 1) << 2) + 2 * hh + (j & 1) : 4 * hh + j;
}

// =============================================================================================
// converter role, FP8 P.V mode (warps 0-11).  Step g: read tile g's FP8 chunks and scales from ring
// stage g % 2, hand the tile's 64 per-token scales and its largest scale to the softmax, release
// the stage; once Q.K^T(g-2) has finished dequantise the K half into buffer g % 2 (as the per-token
// mode does); once P.V(g-2) has finished write tile g's V operand into FP8 buffer g % 2 as raw e4m3
// bytes: the own key's D_c chunks (from the ring reads above) and the other key's D_c chunks
// (loaded from global memory during step g-1).  Then load the other key's chunks of tile g+1.
// =============================================================================================
__device__ __forceinline__ void converter_role_fp8pv(const DecodeParams& p, int k, uint32_t base, int lane,
                                                     volatile uint32_t* abort, uint32_t peer_abort, uint32_t c) {
  const int C = static_cast<int>(c);
  const int t = threadIdx.x;
  const int grp = t / CONV_GROUP, tau = t % CONV_GROUP;
  const int r = conv_row(tau), cq = conv_cq(tau);
  const bool extra = grp == extra_group(C);
  const uint64_t lim = p.wait_limit_ns;
#define BAR(i) (base + SBAR + 8u * (i))
#define MLA_WAIT_RET(b_, parity)                                                               \
  if (!__all_sync(0xffffffffu, wait_bar((b_), (parity), abort, p.status, peer_abort, lim))) return;
#define MLA_POLL_RET(b_, parity)                                                               \
  if (!__all_sync(0xffffffffu, poll_bar((b_), (parity), abort, p.status, peer_abort, lim))) return;
  const uint32_t k_full0 = ptx::mapa(BAR(B_K_FULL), 0), v_full0 = ptx::mapa(BAR(B_V_FULL), 0);
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  const float no_blk[3] = {0.f, 0.f, 0.f};
  TileStream ts(p, k);
  TileInfo kt = ts.take(p);
  if (!kt.valid) return;
  TileInfo nt = ts.take(p);
  Ahead A;
  A.oth_ok = false;
  A.own_ok = true;
  OthLut L = oth_lut_issue(p, kt, C, r);
  if (!fetch_oth<false>(p, L, C, grp, cq, extra, A)) raise_status(p.status, STATUS_BOUNDS);
  if (nt.valid) L = oth_lut_issue(p, nt, C, r);
  uint32_t g = 0;
  while (true) {
    const uint32_t st = g & 1;
    if (t == 0) MLA_TRACE_EV(g, 1);
    MLA_WAIT_RET(BAR(B_RING_FULL + st), (g >> 1) & 1);
    if (t == 0) MLA_TRACE_EV(g, 3);
    const uint32_t stage = base + SRING + st * RING_STAGE;
    const uint32_t mask = ptx::ld_shared_u32(base + S_MASK + 8 * st);
    const uint32_t omask = ptx::ld_shared_u32(base + S_MASK + 8 * st + 4);
    const bool own_ok = ((mask >> r) & 1u) != 0;
    uint4 raw[3];
#pragma unroll
    for (int m = 0; m < 3; ++m) raw[m] = ptx::ld_shared_v4(stage + r * HEAD_DIM + 16 * (4 * (3 * grp + m) + cq));
    const float s_own = ptx::ld_shared_f32(stage + RING_ROWS + 4 * r);
    // the tile's 64 per-token scales and its largest scale for the softmax (slot g % 8; the softmax
    // finished tile g - 8 before S_FREE(g - 5), which Q.K^T(g - 3) waited for before the K-buffer
    // wait of step g - 1 passed)
    if (grp == 0) {
      float mx = 0.f;
      if (cq == 0) {
        const float so = own_ok ? s_own : 0.f;
        const float sx = ((omask >> r) & 1u) ? ptx::ld_shared_f32(stage + RING_OSC + 4 * r) : 0.f;
        const uint32_t sa = base + SSC + (g % SSC_SLOTS) * SSC_STRIDE + 4 * r;
        ptx::st_shared_f32(sa + 4 * HALF_BN * C, so);
        ptx::st_shared_f32(sa + 4 * HALF_BN * (1 - C), sx);
        mx = fmaxf(so, sx);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) ptx::st_shared_f32(base + SSMAX + (g % SSC_SLOTS) * 16 + 4 * (t >> 5), mx);
    }
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive(BAR(B_SC_FULL + (g % SSC_SLOTS)));
      ptx::mbar_arrive(BAR(B_RING_EMPTY + st));    // the reads above are ordered before it
    }
    // K half buffer g % 2: free once Q.K^T(g - 2) has finished
    MLA_POLL_RET(BAR(B_S_FULL + st), ((g >> 1) & 1) ^ 1);
    if (t == 0) MLA_TRACE_EV(g, 16);
    convert_k<false, false>(grp, r, cq, own_ok, raw, s_own, no_blk, base + SK0 + st * SK_STRIDE);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive_cluster(k_full0 + 8u * st);
    if (t == 0) MLA_TRACE_EV(g, 5);
    if (t == 352) MLA_TRACE_EV(g, 26);
    if (lane == 0) MLA_TRACE_EV(g, 32 + (t >> 5));
    // FP8 V buffer g % 2: free once P.V(g - 2) has finished
    if (t == 0) MLA_TRACE_EV(g, 4);
    MLA_WAIT_RET(BAR(B_PV_DONE + st), ((g >> 1) & 1) ^ 1);
    if (t == 0) MLA_TRACE_EV(g, 6);
    {
      const uint32_t sv8 = base + SV + st * SV8_STRIDE;
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        const int a = 3 * grp + m;
        if (!k_in_dc(a, C)) continue;
        const uint4 v = own_ok ? raw[m] : zero4;
        const uint32_t dst = sv8 + (((a >> 1) == C) ? 0u : SV8_ATOM) + sw128_off(HALF_BN * C + r, (a & 1) * 4 + cq);
        ptx::st_shared_v4(dst, v.x, v.y, v.z, v.w);
      }
      const int vrow = HALF_BN * (1 - C) + r;
      {
        const uint4 v = A.oth_ok ? A.oth[0] : zero4;
        ptx::st_shared_v4(sv8 + (grp >> 1) * SV8_ATOM + sw128_off(vrow, (grp & 1) * 4 + cq), v.x, v.y, v.z, v.w);
      }
      if (extra) {
        const uint4 v = A.oth_ok ? A.oth[1] : zero4;
        ptx::st_shared_v4(sv8 + SV8_ATOM + sw128_off(vrow, 4 + cq), v.x, v.y, v.z, v.w);
      }
    }
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive_cluster(v_full0 + 8u * st);
    if (t == 0) MLA_TRACE_EV(g, 2);
    if (t == 352) MLA_TRACE_EV(g, 27);
    if (lane == 0) MLA_TRACE_EV(g, 44 + (t >> 5));
    if (!nt.valid) break;
    if (!fetch_oth<false>(p, L, C, grp, cq, extra, A)) raise_status(p.status, STATUS_BOUNDS);
    if (t == 0) MLA_TRACE_EV(g, 7);
    ++g;
    kt = nt;
    nt = ts.take(p);
    if (nt.valid) L = oth_lut_issue(p, nt, C, r);
  }
#undef MLA_POLL_RET
#undef MLA_WAIT_RET
#undef BAR
}

// =============================================================================================
// producer role (lane 0 of warp 19): walks the cluster's tiles and fills ring stage g % 2 with the
// own keys' rows (and per-token scales) of tile g once the converters have released the stage;
// tile g + 1's page runs are read from the page table before that wait.
// Before returning it waits (bounded, whatever the other roles did) for the copies of the last
// two stages it armed, so that no bulk copy into this CTA's shared memory is in flight at exit.
// =============================================================================================
template <int MODE>
__device__ __forceinline__ void producer_role(const DecodeParams& p, int k, uint32_t base, volatile uint32_t* abort,
                                              uint32_t peer_abort, uint32_t c) {
  constexpr bool SC = MODE != SCALE_BLOCK && MODE != SCALE_BLOCKR;
#define BAR(i) (base + SBAR + 8u * (i))
  TileStream ts(p, k);
  uint32_t g = 0;
  TileInfo ti = ts.take(p);
  StagePlan sp;
  if (ti.valid) sp = plan_stage<SC>(p, item_b(p, ti.item), ti.j, ti.nvis, static_cast<int>(c));
  while (ti.valid) {
    const uint32_t st = g & 1;
    if (!wait_bar(BAR(B_RING_EMPTY + st), ((g >> 1) & 1) ^ 1, abort, p.status, peer_abort, p.wait_limit_ns)) break;
    MLA_TRACE_EV(g, 24);
    if (MODE == SCALE_BLOCKR)
      issue_planned<false, false, true>(p, base + SRING + st * RING_STAGE, BAR(B_RING_FULL + st), base + S_MASK + 8 * st,
                                        sp, base + SBSC + st * BSC_STRIDE);
    else
      issue_planned<SC, SC>(p, base + SRING + st * RING_STAGE, BAR(B_RING_FULL + st), base + S_MASK + 8 * st, sp);
    MLA_TRACE_EV(g, 25);
    ++g;
    // the next tile's page runs (table reads) while stage g % 2 is being read
    ti = ts.take(p);
    if (ti.valid) sp = plan_stage<SC>(p, item_b(p, ti.item), ti.j, ti.nvis, static_cast<int>(c));
  }
  for (uint32_t gd = (g >= 2 ? g - 2 : 0); gd < g; ++gd)
    drain_bar(BAR(B_RING_FULL + (gd & 1)), (gd >> 1) & 1, p.wait_limit_ns);
#undef BAR
}

// =============================================================================================
// decode kernel
// =============================================================================================
// MODE: a ScaleMode (per-token scales, block scales, per-token scales folded into S and P, or the
// e4m3 P.V product).
template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1) mla_decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr bool FOLD = MODE == SCALE_FOLD;
  constexpr bool F8 = MODE == SCALE_FP8PV;
  constexpr bool SCALES = FOLD || F8;   // the converter hands per-token scales to the softmax
  if (threadIdx.x == 0) MLA_MARK_MIN(1);
  ptx::griddep_launch_dependents();   // the combine kernel may start launching (it waits for this grid)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (SCALES && static_cast<uint32_t>(smem - smem_raw) > SMEM_FOLD_MAX_PAD) {
    // every CTA of the launch sees the same base, so all of them leave here together
    if (threadIdx.x == 0) raise_status(p.status, STATUS_LAYOUT);
    return;
  }
  const uint32_t base = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = ptx::cluster_ctarank();
  const uint32_t peer = c ^ 1u;
  const int k = static_cast<int>(ptx::cluster_id_x());
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + S_ABORT);
  const uint32_t peer_abort = ptx::mapa(base + S_ABORT, peer);
  const uint64_t lim = p.wait_limit_ns;
#define BAR(i) (base + SBAR + 8u * (i))
  MLA_TRACE_CTA(0);

  if (threadIdx.x == 0) {
    for (uint32_t i = 0; i < 2; ++i) {
      ptx::mbar_init(BAR(B_K_FULL + i), 2 * CONV_WARPS);
      ptx::mbar_init(BAR(B_V_FULL + i), 2 * CONV_WARPS);
      ptx::mbar_init(BAR(B_PV_DONE + i), 1);
      ptx::mbar_init(BAR(B_S_FULL + i), 1);
      ptx::mbar_init(BAR(B_S_FREE + i), 8);
      ptx::mbar_init(BAR(B_P_FULL + i), 8);
      ptx::mbar_init(BAR(B_RED + 2 * i), 2);
      ptx::mbar_init(BAR(B_RED + 2 * i + 1), 2);
      ptx::mbar_init(BAR(B_REDL + i), 2);
      ptx::mbar_init(BAR(B_RING_FULL + i), 1);
      ptx::mbar_init(BAR(B_RING_EMPTY + i), CONV_WARPS);
    }
    ptx::mbar_init(BAR(B_Q_FULL), 2);
    ptx::mbar_init(BAR(B_Q_FREE), 1);
    ptx::mbar_init(BAR(B_Q_LOCAL), 1);
    ptx::mbar_init(BAR(B_O_FREE), 8);
    ptx::mbar_init(BAR(B_DRAIN), 2);
    ptx::mbar_init(BAR(B_EXIT), 1);
    for (uint32_t i = 0; i < SSC_SLOTS; ++i) ptx::mbar_init(BAR(B_SC_FULL + i), CONV_WARPS);
    *abort = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == QK_WARP) {
    ptx::tmem_alloc_pair(base + S_TMEM_BASE, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // the peer's barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + S_TMEM_BASE);
  ptx::griddep_wait();   // the split plan (previous kernel of the stream) is complete and visible

// Whole-warp roles bail out together so that the warp-collective instructions after a wait never
// run on a partial warp.
#define MLA_WAIT_WARP(b_, parity)                                                              \
  if (!__all_sync(0xffffffffu, wait_bar((b_), (parity), abort, p.status, peer_abort, lim))) goto role_done;
#define MLA_POLL_WARP(b_, parity)                                                              \
  if (!__all_sync(0xffffffffu, poll_bar((b_), (parity), abort, p.status, peer_abort, lim))) goto role_done;

  if (warp < CONV_WARPS) {
    // ------------------------------------------------------------------ converter
    if (F8) converter_role_fp8pv(p, k, base, lane, abort, peer_abort, c);
    else converter_role<MODE>(p, k, base, lane, abort, peer_abort, c);
  } else if (warp < SM_WARP0 + 4) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int t = threadIdx.x - 32 * SM_WARP0;
    const int quad = warp - SM_WARP0;
    const int r = t & 63, hh = t >> 6;             // head row within the CTA, key half of the tile
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t p_full0 = ptx::mapa(BAR(B_P_FULL), 0), s_free0 = ptx::mapa(BAR(B_S_FREE), 0);
    const uint32_t o_free = ptx::mapa(BAR(B_O_FREE), 0);
    volatile float* red_max = reinterpret_cast<volatile float*>(smem + SRED);
    volatile float* red_l = reinterpret_cast<volatile float*>(smem + SRED + 1024);
    UnitWalker wk(p, k);
    Unit u;
    uint32_t g = 0, uu = 0;
    while (wk.next(p, u)) {
      float m_ref = -INFINITY, l = 0.f;
      int sig = 0;   // e4m3 P.V: the unit's weights carry 2^sig (lowered, never raised, as tiles come in)
      for (int j = u.tb; j < u.te; ++j, ++g) {
        const uint32_t sb = g & 1;
        MLA_WAIT_WARP(BAR(B_S_FULL + sb), (g >> 1) & 1);
        if (SCALES) MLA_WAIT_WARP(BAR(B_SC_FULL + (g % SSC_SLOTS)), (g / SSC_SLOTS) & 1);
        if (t == 0) MLA_TRACE_EV(g, 8);
        ptx::tc_fence_after();
        float x[32];
        {
          uint32_t rr[32];
          ptx::tmem_ld32(lane_base + T_S + 32 * sb, rr);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = __uint_as_float(rr[q]);
        }
        // S buffer sb may be overwritten by Q.K^T(g + 2) from here on
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(s_free0 + 8u * sb);
        if (t == 0) MLA_TRACE_EV(g, 9);
        const int nv = min(BN, u.nvis - j * BN) - HALF_BN * hh;   // valid keys in this lane's half
        float mt = -INFINITY;
        // scale-folding and e4m3 P.V modes: the scales of this lane's 32 keys (written before
        // SC_FULL of this tile; slot g % 8 is rewritten only after this warp has finished tile g)
        const uint32_t sc_addr = base + SSC + (g % SSC_SLOTS) * SSC_STRIDE + 4 * HALF_BN * hh;
        // Scores in log2 units are x = S * c (c = scale_log2, times s_t in the scale-folding mode),
        // keys past the request's end at -inf.  The e4m3 P.V mode, whose softmax carries the weight
        // split, saves instructions on whole half-tiles with c > 0 (every tile but a request's
        // last): it keeps x = S, takes the row max as max(S) * c (rounding is monotone) and forms
        // each exponent as one fma(S, c, -m).  (In the other modes the same change costs register
        // spills at this kernel's 96-register limit and measured slower.)
        const float c = p.scale_log2;
        const bool fast = F8 && nv >= HALF_BN && c > 0.f;   // warp-uniform
        if (fast) {
#pragma unroll
          for (int q = 0; q < 32; ++q) mt = fmaxf(mt, x[q]);
          mt *= c;
        } else if (FOLD) {
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 s4 = ptx::ld_shared_v4(sc_addr + 16 * v);
            const float sc[4] = {__uint_as_float(s4.x), __uint_as_float(s4.y), __uint_as_float(s4.z),
                                 __uint_as_float(s4.w)};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = 4 * v + e;
              x[q] = (q < nv) ? x[q] * (c * sc[e]) : -INFINITY;
              mt = fmaxf(mt, x[q]);
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            x[q] = (q < nv) ? x[q] * c : -INFINITY;
            mt = fmaxf(mt, x[q]);
          }
        }
        // the other half of this head row lives in lane t ^ 64 (another warp of this warpgroup)
        red_max[sb * 128 + t] = mt;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(BAR(B_RED + 2 * sb + (quad & 1)));
        MLA_WAIT_WARP(BAR(B_RED + 2 * sb + (quad & 1)), (g >> 1) & 1);
        mt = fmaxf(mt, red_max[sb * 128 + (t ^ 64)]);
        if (t == 0) MLA_TRACE_EV(g, 10);
        float alpha = 1.f;
        bool rescale = false;
        // lazy max: keep the reference unless it grows by more than 8 (2 for e4m3 weights) in log2 units
        if (mt > m_ref + (F8 ? FP8_PV_LAZY_LOG2 : 8.f)) {
          alpha = (m_ref == -INFINITY) ? 0.f : ptx::ex2_approx(m_ref - mt);
          l *= alpha;
          rescale = (j != u.tb);
          m_ref = mt;
        }
        // e4m3 P.V: sigma of this tile's largest scale; a drop scales O by 2^(new - old) as well
        float sfac = 1.f;
        if (F8) {
          const uint4 m4 = ptx::ld_shared_v4(base + SSMAX + (g % SSC_SLOTS) * 16);
          const float smx = fmaxf(fmaxf(__uint_as_float(m4.x), __uint_as_float(m4.y)),
                                  fmaxf(__uint_as_float(m4.z), __uint_as_float(m4.w)));
          const int st = fp8_pv_sigma(smx);
          if (j == u.tb) {
            sig = st;
          } else if (st < sig) {
            sfac = exp2i_or_zero(st - sig);
            sig = st;
          }
        }
        float lsum = 0.f;
        uint32_t pw[16];
        const float cmul = fast ? c : 1.f;
        if (F8) {
          // P carries w = p * s_t * 2^sig as two e4m3 terms (p <= 4 under the lazy max, s_t * 2^sig
          // <= 112, so w <= 448).  The exponent takes 2^sig in (p' = 2^(x - m + sig)); l sums p'
          // and is scaled back by 2^-sig once per tile.
          const float mo = m_ref - static_cast<float>(sig);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 s4 = ptx::ld_shared_v4(sc_addr + 16 * v);
            const float p0 = ptx::ex2_approx(fmaf(x[4 * v], cmul, -mo));
            const float p1 = ptx::ex2_approx(fmaf(x[4 * v + 1], cmul, -mo));
            const float p2 = ptx::ex2_approx(fmaf(x[4 * v + 2], cmul, -mo));
            const float p3 = ptx::ex2_approx(fmaf(x[4 * v + 3], cmul, -mo));
            lsum += p0 + p1;
            lsum += p2 + p3;
            uint32_t h01, l01, h23, l23;
            split2_e4m3(p0 * __uint_as_float(s4.x), p1 * __uint_as_float(s4.y), h01, l01);
            split2_e4m3(p2 * __uint_as_float(s4.z), p3 * __uint_as_float(s4.w), h23, l23);
            pw[v] = h01 | (h23 << 16);
            pw[8 + v] = l01 | (l23 << 16);
          }
          lsum *= exp2i(-sig);
        } else if (FOLD) {
          // l sums the weights; the P operand carries weight * s_t
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 s4 = ptx::ld_shared_v4(sc_addr + 16 * v);
            const float p0 = ptx::ex2_approx(x[4 * v] - m_ref);
            const float p1 = ptx::ex2_approx(x[4 * v + 1] - m_ref);
            const float p2 = ptx::ex2_approx(x[4 * v + 2] - m_ref);
            const float p3 = ptx::ex2_approx(x[4 * v + 3] - m_ref);
            lsum += p0 + p1;                // the per-token mode's summation order
            lsum += p2 + p3;
            pw[2 * v] = ptx::pack_bf16x2(p0 * __uint_as_float(s4.x), p1 * __uint_as_float(s4.y));
            pw[2 * v + 1] = ptx::pack_bf16x2(p2 * __uint_as_float(s4.z), p3 * __uint_as_float(s4.w));
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float p0 = ptx::ex2_approx(x[2 * q] - m_ref);
            const float p1 = ptx::ex2_approx(x[2 * q + 1] - m_ref);
            lsum += p0 + p1;
            pw[q] = ptx::pack_bf16x2(p0, p1);
          }
        }
        l += lsum;
        if (t == 0) MLA_TRACE_EV(g, 11);
        // the P buffer is free once P.V(g - 1) has finished (O may be rescaled from then on too)
        if (g > 0) MLA_WAIT_WARP(BAR(B_PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1);
        if (t == 0) MLA_TRACE_EV(g, 13);
        {
          const uint32_t sp = base + SP;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            ptx::st_shared_v4(sp + sw128_off(r, p_unit<F8>(hh, v)), pw[4 * v], pw[4 * v + 1], pw[4 * v + 2],
                              pw[4 * v + 3]);
        }
        // O rescale (warp-collective TMEM access): a warp rescales when any of its rows moved its
        // reference max (or sigma dropped); rows that did not move use alpha = 1
        if (!rescale) alpha = 1.f;
        alpha *= sfac;
        if (__any_sync(0xffffffffu, rescale) || sfac != 1.f) {
          ptx::tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t rr[32];
            ptx::tmem_ld32(lane_base + T_O + 32 * ch, rr);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) rr[q] = __float_as_uint(__uint_as_float(rr[q]) * alpha);
            ptx::tmem_st32(lane_base + T_O + 32 * ch, rr);
          }
          ptx::tmem_wait_st();
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(p_full0 + 8u * sb);
        if (t == 0) MLA_TRACE_EV(g, 14);
      }
      // epilogue: O / l for this lane's 256 V dims of head row r
      {
        const uint32_t gl = g - 1;
        if (gl > 0) MLA_WAIT_WARP(BAR(B_PV_DONE + ((gl - 1) & 1)), ((gl - 1) >> 1) & 1);
        MLA_WAIT_WARP(BAR(B_PV_DONE + (gl & 1)), (gl >> 1) & 1);
        ptx::tc_fence_after();
        red_l[t] = l;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(BAR(B_REDL + (quad & 1)));
        MLA_WAIT_WARP(BAR(B_REDL + (quad & 1)), uu & 1);
        const float l_row = l + red_l[t ^ 64];
        const float inv_l = F8 ? exp2i(-sig) / l_row : 1.f / l_row;
        const int head = u.g * MROWS + HPC * static_cast<int>(c) + r;
        const bool row_ok = head < p.H;
        const float lse_v = (m_ref + ptx::lg2_approx(l_row)) * 0.69314718055994530942f;
        // O / l goes out through the P buffer, idle once the unit's last P.V has finished: each
        // thread stages 64 bytes of its row (32 bf16, or 16 fp32 per half of a chunk) in the four
        // 16-byte units of its own P row that it writes as P, then the warp stores whole 64-byte row
        // segments.  A warp touches only its own P units, so a warp still in its epilogue is not
        // disturbed by one that has begun the next unit.  The read-back takes rows x and x ^ PX in
        // one 8-thread phase (PX = 4 for bf16 P, 2 for e4m3 P): their units sit in opposite halves
        // of the swizzle row, so both passes are conflict-free.
        const uint32_t sp = base + SP;
        const int prow0 = 32 * (quad & 1);                                // P row of this warp's lane 0
        const int row0 = HPC * static_cast<int>(c) + prow0;               // CTA row of this warp's lane 0
        constexpr int PXB = F8 ? 1 : 2;
        const int rb_j = lane & 3;
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t rr[32];
          ptx::tmem_ld32(lane_base + T_O + 32 * ch, rr);
          ptx::tmem_wait_ld();
          const int dv = (ch < 4 ? 0 : 256) + 128 * hh + 32 * (ch & 3);
          if (u.slot < 0) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t w0 = ptx::pack_bf16x2(__uint_as_float(rr[8 * v + 0]) * inv_l, __uint_as_float(rr[8 * v + 1]) * inv_l);
              const uint32_t w1 = ptx::pack_bf16x2(__uint_as_float(rr[8 * v + 2]) * inv_l, __uint_as_float(rr[8 * v + 3]) * inv_l);
              const uint32_t w2 = ptx::pack_bf16x2(__uint_as_float(rr[8 * v + 4]) * inv_l, __uint_as_float(rr[8 * v + 5]) * inv_l);
              const uint32_t w3 = ptx::pack_bf16x2(__uint_as_float(rr[8 * v + 6]) * inv_l, __uint_as_float(rr[8 * v + 7]) * inv_l);
              ptx::st_shared_v4(sp + sw128_off(prow0 + lane, p_unit<F8>(hh, v)), w0, w1, w2, w3);
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int n = 4 * it + (lane >> 3), j = rb_j;
              const int x = ((n >> PXB) << (PXB + 1)) | (n & ((1 << PXB) - 1)) | (((lane >> 2) & 1) << PXB);
              const uint4 w = ptx::ld_shared_v4(sp + sw128_off(prow0 + x, p_unit<F8>(hh, j)));
              const int hd = u.g * MROWS + row0 + x;
              if (hd < p.H)
                *reinterpret_cast<uint4*>(p.out + ((static_cast<size_t>(u.b) * p.T + u.i) * p.H + hd) * V_DIM + dv + 8 * j) = w;
            }
          } else {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                ptx::st_shared_v4(sp + sw128_off(prow0 + lane, p_unit<F8>(hh, v)),
                                  __float_as_uint(__uint_as_float(rr[16 * hf + 4 * v + 0]) * inv_l),
                                  __float_as_uint(__uint_as_float(rr[16 * hf + 4 * v + 1]) * inv_l),
                                  __float_as_uint(__uint_as_float(rr[16 * hf + 4 * v + 2]) * inv_l),
                                  __float_as_uint(__uint_as_float(rr[16 * hf + 4 * v + 3]) * inv_l));
              __syncwarp();
#pragma unroll
              for (int it = 0; it < 4; ++it) {
                const int n = 4 * it + (lane >> 3), j = rb_j;
                const int x = ((n >> PXB) << (PXB + 1)) | (n & ((1 << PXB) - 1)) | (((lane >> 2) & 1) << PXB);
                const uint4 w = ptx::ld_shared_v4(sp + sw128_off(prow0 + x, p_unit<F8>(hh, j)));
                *reinterpret_cast<uint4*>(p.part_o + (static_cast<size_t>(u.slot) * MROWS + row0 + x) * V_DIM + dv +
                                          16 * hf + 4 * j) = w;
              }
              __syncwarp();
            }
          }
          __syncwarp();
        }
        if (hh == 0 && row_ok) {
          if (u.slot < 0) {
            if (p.lse) p.lse[(static_cast<size_t>(u.b) * p.T + u.i) * p.H + head] = lse_v;
          } else {
            p.part_lse[static_cast<size_t>(u.slot) * MROWS + HPC * c + r] = lse_v;
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(o_free);
        if (t == 0) MLA_TRACE_EV(g - 1, 15);
      }
      ++uu;
    }
  } else if (warp == Q_WARP) {
    // ------------------------------------------------------------------ Q loader (both CTAs)
    // Per unit: wait until the last Q.K^T of the previous unit has finished, then one TMA load per
    // 64-dim atom column of the CTA's 64 heads (heads past H read as zero).  The load's own
    // barrier is always waited for (time-bounded, whatever the other roles did), so no TMA write
    // into this CTA's shared memory is in flight when it exits.
    if (lane == 0) {
      const uint32_t q_full = ptx::mapa(BAR(B_Q_FULL), 0);
      ptx::prefetch_tmap(&p.tmap_q);
      UnitWalker wk(p, k);
      Unit u;
      uint32_t uu = 0;
      while (wk.next(p, u)) {
        if (!wait_bar(BAR(B_Q_FREE), (uu & 1) ^ 1, abort, p.status, peer_abort, lim)) break;
        ptx::mbar_arrive_expect_tx(BAR(B_Q_LOCAL), 9 * SQ_ATOM);
#pragma unroll 1
        for (int a = 0; a < 9; ++a)
          ptx::tma_load_3d(base + SQ + a * SQ_ATOM, &p.tmap_q, 64 * a, u.g * MROWS + HPC * static_cast<int>(c),
                           u.b * p.T + u.i, BAR(B_Q_LOCAL));
        drain_bar(BAR(B_Q_LOCAL), uu & 1, lim);
        if (*abort) break;
        const bool withhold = p.inject == INJECT_SKIP_Q_ARRIVAL && k == 0 && c == 1 && uu == 0;
        if (!withhold) ptx::mbar_arrive_cluster(q_full);
        ++uu;
      }
      // drain: the last unit's Q_FREE commit lands in this CTA before it exits
      if (uu > 0) wait_bar(BAR(B_Q_FREE), (uu & 1) ^ 1, abort, p.status, peer_abort, lim);
    }
  } else if (warp == LOAD_WARP) {
    // ------------------------------------------------------------------ FP8 producer (both CTAs)
    if (lane == 0) producer_role<MODE>(p, k, base, abort, peer_abort, c);
  } else if (warp == QK_WARP) {
    // ------------------------------------------------------------------ Q.K^T issuer (CTA 0)
    // The whole warp runs the loop (descriptors stay warp-uniform); one elected lane issues.
    if (c == 0) {
      TileCursor qc(p, k);
      uint32_t g = 0, uq = 0;
      // descriptor bases; per K step only the start-address field (bits 0..13, bytes >> 4) moves
      const uint64_t dq0 = ptx::smem_desc(base + SQ, 16, 1024, ptx::SW_128B);
      const uint64_t dk0 = ptx::smem_desc(base + SK0, 16, 1024, ptx::SW_128B);
      while (qc.valid) {
        const uint32_t sb = g & 1;
        if (qc.first) {
          // the unit's Q is in shared memory (both CTAs); its first 384 dims go to tensor memory
          // once, so that the Q.K^T MMAs of the unit read that part of A from there.  The previous
          // unit's MMAs have finished (the Q loader waited for Q_FREE before loading).
          MLA_POLL_WARP(BAR(B_Q_FULL), uq & 1);
          ++uq;
          ptx::tc_fence_after();
          if (ptx::elect_one()) {
#pragma unroll 1
            for (int a = 0; a < Q_TMEM_ATOMS; ++a)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                ptx::tmem_cp_pair_64x128_dup(tbase + T_Q + 32 * a + 4 * j,
                                             ptx::smem_desc(base + SQ + a * SQ_ATOM + 16 * j, 16, 1024, ptx::SW_128B));
          }
          __syncwarp();
        }
        MLA_POLL_WARP(BAR(B_K_FULL + sb), (g >> 1) & 1);
        MLA_POLL_WARP(BAR(B_S_FREE + sb), ((g >> 1) & 1) ^ 1);
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          MLA_TRACE_EV(g, 20);
          const uint32_t dS = tbase + T_S + 32 * sb;
          // 9 atom columns of 64 dims x 4 K steps of 16 dims: A from tensor memory for atom
          // columns 0..5 (8 columns per K step), from shared memory for 6..8
          uint64_t bd = dk0 + ((sb * SK_STRIDE) >> 4);
#pragma unroll 1
          for (int a = 0; a < Q_TMEM_ATOMS; ++a) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_pair_ts(dS, tbase + T_Q + 32 * a + 8 * kk, bd + kk * 2, IDESC_QK, (a | kk) != 0 ? 1u : 0u);
            bd += SK_ATOM >> 4;
          }
          uint64_t ad = dq0 + ((Q_TMEM_ATOMS * SQ_ATOM) >> 4);
#pragma unroll 1
          for (int a = Q_TMEM_ATOMS; a < 9; ++a) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) ptx::mma_pair_ss(dS, ad + kk * 2, bd + kk * 2, IDESC_QK, 1u);
            ad += SQ_ATOM >> 4;
            bd += SK_ATOM >> 4;
          }
          ptx::mma_commit_pair(BAR(B_S_FULL + sb), 0x3);
          MLA_TRACE_EV(g, 21);
          if (qc.j == qc.u.te - 1) ptx::mma_commit_pair(BAR(B_Q_FREE), 0x3);
        }
        __syncwarp();
        ++g;
        qc.advance(p);
      }
      // drain: the S_FREE arrivals of the last two tiles (nothing else waits for them)
      for (uint32_t gd = (g >= 2 ? g - 2 : 0); gd < g; ++gd) MLA_POLL_WARP(BAR(B_S_FREE + (gd & 1)), (gd >> 1) & 1);
    }
  } else if (warp == PV_WARP) {
    // ------------------------------------------------------------------ P.V issuer (CTA 0)
    if (c == 0) {
      TileCursor pc(p, k);
      uint32_t g = 0, up = 0;
      const uint64_t dp0 = ptx::smem_desc(base + SP, 16, 1024, ptx::SW_128B);
      const uint64_t dv0 = ptx::smem_desc(base + SV, F8 ? SV8_ATOM : SV_ATOM, 1024, ptx::SW_128B);
      while (pc.valid) {
        const uint32_t hb = g & 1;
        const bool first = pc.first;
        MLA_POLL_WARP(BAR(B_V_FULL + hb), (g >> 1) & 1);
        MLA_POLL_WARP(BAR(B_P_FULL + hb), (g >> 1) & 1);
        if (first) {
          MLA_POLL_WARP(BAR(B_O_FREE), (up & 1) ^ 1);
          ++up;
        }
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          MLA_TRACE_EV(g, 22);
          if (F8) {
            // e4m3: per 128-dim half jv, (hi, lo) x two 32-key K steps; A = P bytes 0..63 (hi) and
            // 64..127 (lo) of each head row, B = V buffer g % 2 (one 128-dim atom column per CTA)
#pragma unroll
            for (int jv = 0; jv < 2; ++jv) {
#pragma unroll
              for (int tm = 0; tm < 2; ++tm) {
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                  const uint64_t ad = dp0 + ((64 * tm + 32 * kb) >> 4);
                  const uint64_t bd = dv0 + ((hb * SV8_STRIDE + jv * SV8_ATOM + kb * 4096) >> 4);
                  ptx::mma_pair_ss_f8(tbase + T_O + 128 * jv, ad, bd, IDESC_PV8, (first && (tm | kb) == 0) ? 0u : 1u);
                }
              }
            }
          } else {
#pragma unroll
            for (int jv = 0; jv < 2; ++jv) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = dp0 + ((kk * 32) >> 4);
                const uint64_t bd = dv0 + ((2 * jv * SV_ATOM + kk * 2048) >> 4);
                ptx::mma_pair_ss(tbase + T_O + 128 * jv, ad, bd, IDESC_PV, (first && kk == 0) ? 0u : 1u);
              }
            }
          }
          ptx::mma_commit_pair(BAR(B_PV_DONE + hb), 0x3);
          MLA_TRACE_EV(g, 23);
        }
        __syncwarp();
        ++g;
        pc.advance(p);
      }
      // drain: the last unit's O_FREE arrivals (both CTAs' epilogues)
      if (up > 0) MLA_POLL_WARP(BAR(B_O_FREE), (up - 1) & 1);
    }
  }
role_done:
#undef MLA_POLL_WARP
#undef MLA_WAIT_WARP
  // Every pair MMA issued by CTA 0 has finished before TMEM is released.  The commit arrives once
  // all of the issuer's earlier MMAs are done; the MMAs themselves wait on nothing, so on a normal
  // or an aborted call this wait ends well inside its bound (it only bounds the spin).
  if (c == 0 && (warp == QK_WARP || warp == PV_WARP) && lane == 0) {
    ptx::mma_commit_pair(BAR(B_DRAIN), 0x1);
    drain_bar(BAR(B_DRAIN), 0, lim);
  }
  ptx::tc_fence_before();
  __syncthreads();
  MLA_TRACE_CTA(2);
  // Exit handshake.  Every cross-CTA arrival and pair-MMA commit has been waited for above, so no
  // remote access can reach a CTA that has exited; the two CTAs still tell each other that they are
  // done (one remote arrive each) before the pair's TMEM is released.  The arrive releases at
  // cluster scope, after the CTA barrier above, so every remote arrival this CTA's threads made
  // earlier (also on an aborted call, where nothing on the peer waited for them) reaches the peer
  // before the peer can exit.  The wait polls: a thread suspended in try_wait (or in a cluster
  // barrier) measured ~7 us to resume after the peer's remote arrival on B200, even with both
  // CTAs arriving together.
  if (threadIdx.x == 0) {
    ptx::mbar_arrive_remote(ptx::mapa(BAR(B_EXIT), peer));
#ifdef MLA_TRACE
    if (p.trace) p.trace[2 * TRACE_TILES * TRACE_EVENTS + 4 * blockIdx.x + 1] = ptx::globaltimer();
#endif
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_test_wait(BAR(B_EXIT), 0) && ptx::globaltimer() - t0 < lim) __nanosleep(32);
  }
  __syncthreads();
#undef BAR
  if (warp == QK_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tbase, TMEM_COLS);
    if (lane == 0) MLA_MARK_MAX(2);
#ifdef MLA_TRACE
    if (lane == 0 && p.trace) p.trace[2 * TRACE_TILES * TRACE_EVENTS + 4 * blockIdx.x + 3] = ptx::globaltimer();
#endif
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
  ptx::griddep_launch_dependents();   // the decode kernel may launch and run its prologue meanwhile
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
  __syncthreads();
  if (t == 0) MLA_MARK_MAX(0);
}

// =============================================================================================
// split-KV combine: lse = log sum_s e^{lse_s}; out = sum_s e^{lse_s - lse} out_s  (one warp per head)
// =============================================================================================
constexpr int COMBINE_HEADS = 8;

__global__ void __launch_bounds__(32 * COMBINE_HEADS)
mla_combine_kernel(const __grid_constant__ DecodeParams p) {
  if (threadIdx.x == 0) MLA_MARK_MIN(5);
  ptx::griddep_wait();   // the decode kernel's partials are complete and visible
  if (threadIdx.x == 0) MLA_MARK_MIN(3);
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
  const int bi = static_cast<int>(p.divG.div(it));
  const int g = it - bi * p.G, b = static_cast<int>(p.divT.div(bi)), i = bi - b * p.T;
  const int head = g * MROWS + h;
  if (head >= p.H) return;
  // one pass over the pieces, merging with a running maximum (each piece's LSE and data are loaded
  // together, so the pieces' loads overlap)
  float mx = -INFINITY, tot = 0.f;
  float4 acc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int kk = k0; kk <= k1; ++kk) {
    const int slot = 2 * kk + (max(s, kk * tpc) == kk * tpc ? 0 : 1);
    const float l = p.part_lse[slot * MROWS + h];
    const float4* src = reinterpret_cast<const float4*>(p.part_o + (static_cast<size_t>(slot) * MROWS + h) * V_DIM);
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = src[j * 32 + lane];
    const float mn = fmaxf(mx, l);
    const float a = __expf(mx - mn), wgt = __expf(l - mn);   // a = 0 for the first piece
    mx = mn;
    tot = tot * a + wgt;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[j].x = acc[j].x * a + wgt * v[j].x;
      acc[j].y = acc[j].y * a + wgt * v[j].y;
      acc[j].z = acc[j].z * a + wgt * v[j].z;
      acc[j].w = acc[j].w * a + wgt * v[j].w;
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
  if (lane == 0) MLA_MARK_MAX(4);
}

// =============================================================================================
// gather + dequant kernel (steps A and C alone): one CTA of 384 threads per (request, 64-key tile,
// key half c).  Runs the decode's producer (issue_stage: page runs -> one ring stage) and its
// converter (fetch_own_scales for block scales, convert_k), then copies the K-half buffer out.
// =============================================================================================
constexpr int DQ_THREADS = CONV_THREADS;
constexpr uint32_t DQ_SK = 0;
constexpr uint32_t DQ_RING = SK_STRIDE;
constexpr uint32_t DQ_BAR = DQ_RING + RING_STAGE;
constexpr uint32_t DQ_SMEM_ALLOC = DQ_BAR + 64 + 1024;

template <bool BS>
__global__ void __launch_bounds__(DQ_THREADS)
mla_dequant_kernel(const __grid_constant__ DecodeParams p, const uint32_t* cache_lengths, int max_keys,
                   int tiles_per_req, uint16_t* out_k) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = ptx::smem_u32(smem);
  const int b = blockIdx.x / tiles_per_req;
  const int j = blockIdx.x % tiles_per_req;
  const int c = blockIdx.y;
  if (b >= p.B) return;
  const int n = min(static_cast<int>(min(cache_lengths[b], 0x3FFFFFFFu)) + p.T, max_keys);
  const int tok0 = j * BN + HALF_BN * c;
  if (tok0 >= n) return;
  const int cnt = min(HALF_BN, n - tok0);
  const uint32_t full = base + DQ_BAR, mask_addr = base + DQ_BAR + 8;
  if (threadIdx.x == 0) {
    ptx::mbar_init(full, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) issue_stage<!BS, false>(p, base + DQ_RING, full, mask_addr, b, j, n, c);
  const int t = threadIdx.x, grp = t / CONV_GROUP, tau = t % CONV_GROUP;
  const int r = conv_row(tau), cq = conv_cq(tau);
  Ahead A;
  A.own_ok = true;
  if (BS) {
    TileInfo ti;
    ti.item = b * p.T * p.G;
    ti.nvis = n;
    ti.j = j;
    ti.first = true;
    ti.valid = true;
    if (!fetch_own_scales(p, ti, c, grp, r, cq, A)) raise_status(p.status, STATUS_BOUNDS);
  }
  const uint64_t t0 = ptx::globaltimer();
  bool landed;
  while (!(landed = ptx::mbar_try_wait(full, 0)) && ptx::globaltimer() - t0 < p.wait_limit_ns) {}
  if (!landed) raise_status(p.status, STATUS_TIMEOUT);
  const bool own_ok = landed && ((ptx::ld_shared_u32(mask_addr) >> r) & 1u) != 0 && A.own_ok;
  uint4 raw[3];
#pragma unroll
  for (int m = 0; m < 3; ++m) raw[m] = ptx::ld_shared_v4(base + DQ_RING + r * HEAD_DIM + 16 * (4 * (3 * grp + m) + cq));
  const float s_own = BS ? 0.f : ptx::ld_shared_f32(base + DQ_RING + RING_ROWS + 4 * r);
  convert_k<BS, false>(grp, r, cq, own_ok, raw, s_own, A.s_own, base + DQ_SK);
  __syncthreads();
  for (int id = threadIdx.x; id < HALF_BN * 72; id += DQ_THREADS) {
    const int row = id / 72, cc = id - row * 72;        // 72 units of 8 bf16 per key
    if (row >= cnt) continue;
    const uint4 v = ptx::ld_shared_v4(base + DQ_SK + (cc >> 3) * SK_ATOM + sw128_off(row, cc & 7));
    uint16_t* dst = out_k + (static_cast<size_t>(b) * max_keys + tok0 + row) * HEAD_DIM + cc * 8;
    *reinterpret_cast<uint4*>(dst) = v;
  }
}

}  // namespace mla
