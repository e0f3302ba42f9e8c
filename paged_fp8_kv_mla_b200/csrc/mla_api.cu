// Host side of the C ABI declared in include/mla_paged_fp8.h: argument validation, the
// per-device workspace, and the three launches (plan -> decode -> combine) on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "mla_kernels.cuh"
#include "mla_kv_store.cuh"
#include "mla_merge.cuh"
#include "mla_paged_fp8.h"

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_ev_before = nullptr;
thread_local cudaEvent_t g_ev_after = nullptr;
#ifdef MLA_TRACE
unsigned long long* g_trace = nullptr;
#endif

mla_status_t fail(mla_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define MLA_CUDA(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(MLA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

// ---------------------------------------------------------------- workspace (per device)
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
Workspace g_ws[kMaxDevices];
int g_default_nc[kMaxDevices];         // resident 2-CTA cluster slots, 0 = not queried yet
bool g_attr_set[kMaxDevices];
int g_forced_nc = 0;
unsigned long long g_wait_limit_ns = mla::DEFAULT_WAIT_LIMIT_NS;
int g_inject_once = mla::INJECT_NONE;   // test hook, consumed by the next decode call

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
  size_t hdr, item_start, item_nvis, cluster_first, part_lse, part_o, total;
};

WsLayout ws_layout(int items, int NC) {
  WsLayout L{};
  size_t o = 0;
  L.hdr = o;           o = align_up(o + 64, 256);
  L.item_start = o;    o = align_up(o + sizeof(int32_t) * (items + 1), 256);
  L.item_nvis = o;     o = align_up(o + sizeof(int32_t) * items, 256);
  L.cluster_first = o; o = align_up(o + sizeof(int32_t) * NC, 256);
  L.part_lse = o;      o = align_up(o + sizeof(float) * 2 * NC * mla::MROWS, 256);
  L.part_o = o;        o = align_up(o + sizeof(float) * 2 * NC * mla::MROWS * mla::V_DIM, 256);
  L.total = o;
  return L;
}

mla_status_t ensure_workspace(int dev, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[dev];
  if (w.bytes < bytes) {
    if (w.ptr) {
      MLA_CUDA(cudaDeviceSynchronize());
      MLA_CUDA(cudaFree(w.ptr));
      w.ptr = nullptr;
      w.bytes = 0;
    }
    const size_t want = align_up(bytes + bytes / 4, 1 << 20);
    cudaError_t e = cudaMalloc(&w.ptr, want);
    if (e != cudaSuccess) {
      w.ptr = nullptr;
      return fail(MLA_ERR_WORKSPACE, "workspace cudaMalloc(%zu) failed: %s", want, cudaGetErrorString(e));
    }
    w.bytes = want;
  }
  *out = w.ptr;
  return MLA_OK;
}

mla_status_t device_setup(int dev, int* nc_out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_attr_set[dev]) {
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_decode_kernel<mla::SCALE_TOKEN>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mla::SMEM_ALLOC)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_decode_kernel<mla::SCALE_BLOCK>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mla::SMEM_ALLOC)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_decode_kernel<mla::SCALE_FOLD>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mla::SMEM_ALLOC_FOLD)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_decode_kernel<mla::SCALE_FP8PV>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mla::SMEM_ALLOC_FOLD)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_decode_kernel<mla::SCALE_BLOCKR>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mla::SMEM_ALLOC_FOLD)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_dequant_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(mla::DQ_SMEM_ALLOC)));
    MLA_CUDA(cudaFuncSetAttribute(mla::mla_dequant_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(mla::DQ_SMEM_ALLOC)));
    g_attr_set[dev] = true;
  }
  if (g_default_nc[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 1024);
    cfg.blockDim = dim3(mla::NUM_THREADS);
    cfg.dynamicSmemBytes = mla::SMEM_ALLOC;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0, n_bs = 0, n_fold = 0, n_f8 = 0, n_bsr = 0;
    MLA_CUDA(cudaOccupancyMaxActiveClusters(&n, mla::mla_decode_kernel<mla::SCALE_TOKEN>, &cfg));
    MLA_CUDA(cudaOccupancyMaxActiveClusters(&n_bs, mla::mla_decode_kernel<mla::SCALE_BLOCK>, &cfg));
    cfg.dynamicSmemBytes = mla::SMEM_ALLOC_FOLD;
    MLA_CUDA(cudaOccupancyMaxActiveClusters(&n_fold, mla::mla_decode_kernel<mla::SCALE_FOLD>, &cfg));
    MLA_CUDA(cudaOccupancyMaxActiveClusters(&n_f8, mla::mla_decode_kernel<mla::SCALE_FP8PV>, &cfg));
    MLA_CUDA(cudaOccupancyMaxActiveClusters(&n_bsr, mla::mla_decode_kernel<mla::SCALE_BLOCKR>, &cfg));
    n = n < n_bs ? n : n_bs;
    n = n < n_fold ? n : n_fold;
    n = n < n_f8 ? n : n_f8;
    n = n < n_bsr ? n : n_bsr;
    if (n <= 0) return fail(MLA_ERR_UNSUPPORTED, "no 2-CTA cluster of the decode kernel fits on this device");
    g_default_nc[dev] = n;
  }
  *nc_out = g_forced_nc > 0 ? g_forced_nc : g_default_nc[dev];
  return MLA_OK;
}

// Multiplier and shifts of mla::FastDiv for divisor d >= 1 (l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1).
mla::FastDiv make_fastdiv(uint32_t d) {
  mla::FastDiv f{};
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  f.d = d;
  f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
  f.s1 = l < 1 ? l : 1;
  f.s2 = l > 0 ? l - 1 : 0;
  return f;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared validation of the cache description; fills the parts of DecodeParams that describe it.
mla_status_t check_cache(const void* blocks, const float* scales, const uint32_t* cache_lengths,
                         const uint32_t* lookup_table, uint32_t max_prompt_length, uint32_t max_cache_length,
                         uint32_t layer_idx, const mla_paged_shape_t* s, mla::DecodeParams* p, uint64_t* rows) {
  if (!s) return fail(MLA_ERR_INVALID_ARG, "shape is NULL");
  if (!blocks || !scales || !cache_lengths || !lookup_table)
    return fail(MLA_ERR_INVALID_ARG, "blocks, scales, cache_lengths and lookup_table must be non-NULL");
  if (s->batch < 0 || s->num_q_heads < 1 || s->num_blocks < 1 || s->kv_dim < 1 || s->num_layers < 1 ||
      s->page_size < 1 || s->num_kv_heads < 1 || s->num_scale_blocks < 1 || s->head_dim_granularity < 1 ||
      s->max_pages < 1)
    return fail(MLA_ERR_INVALID_ARG, "non-positive dimension in shape");
  if (s->head_dim != mla::HEAD_DIM || s->v_dim != mla::V_DIM)
    return fail(MLA_ERR_UNSUPPORTED, "head_dim must be 576 and v_dim 512 (got %d, %d)", s->head_dim, s->v_dim);
  if (s->num_kv_heads != 1) return fail(MLA_ERR_UNSUPPORTED, "num_kv_heads must be 1 (MLA latent cache)");
  const int g = s->head_dim_granularity;
  if (mla::HEAD_DIM % g != 0 || (mla::HEAD_DIM / g) % 16 != 0)
    return fail(MLA_ERR_UNSUPPORTED,
                "head_dim_granularity %d: each scale must cover a multiple of 16 of the 576 dims "
                "(1, 2, 3, 4, 6, 9, 12, 18 or 36)", g);
  if (s->page_size % 16 != 0) return fail(MLA_ERR_UNSUPPORTED, "page_size must be a multiple of 16");
  if (layer_idx >= static_cast<uint32_t>(s->num_layers))
    return fail(MLA_ERR_INVALID_ARG, "layer_idx %u >= num_layers %d", layer_idx, s->num_layers);
  if (max_prompt_length < 1) return fail(MLA_ERR_INVALID_ARG, "max_prompt_length must be >= 1");
  if (!aligned16(blocks) || !aligned16(scales)) return fail(MLA_ERR_INVALID_ARG, "blocks and scales must be 16-byte aligned");
  const uint64_t r = static_cast<uint64_t>(s->num_blocks) * s->kv_dim * s->num_layers * s->page_size;
  const uint64_t sr = static_cast<uint64_t>(s->num_scale_blocks) * s->kv_dim * s->num_layers * s->page_size;
  if (r >= (1ull << 31) || sr >= (1ull << 32))
    return fail(MLA_ERR_UNSUPPORTED, "block pool too large (%llu rows)", static_cast<unsigned long long>(r));
  const uint64_t need_pages = (static_cast<uint64_t>(max_cache_length) + max_prompt_length + s->page_size - 1) / s->page_size;
  if (need_pages > static_cast<uint64_t>(s->max_pages))
    return fail(MLA_ERR_INVALID_ARG, "lookup_table has %d pages per request, %llu needed for max_cache_length %u",
                s->max_pages, static_cast<unsigned long long>(need_pages), max_cache_length);
  if (static_cast<uint64_t>(max_cache_length) + max_prompt_length + 64 >= (1ull << 30))
    return fail(MLA_ERR_UNSUPPORTED, "max_cache_length too large");
  p->scales = scales;
  p->lut = lookup_table;
  p->B = s->batch;
  p->T = static_cast<int>(max_prompt_length);
  p->H = s->num_q_heads;
  p->G = (s->num_q_heads + mla::MROWS - 1) / mla::MROWS;
  p->P = s->page_size;
  p->KVD = s->kv_dim;
  p->NL = s->num_layers;
  p->layer = static_cast<int>(layer_idx);
  p->NB = s->num_blocks;
  p->NSB = s->num_scale_blocks;
  p->max_pages = s->max_pages;
  p->blocks = static_cast<const uint8_t*>(blocks);
  p->divP = make_fastdiv(static_cast<uint32_t>(p->P));
  p->SG = s->head_dim_granularity;
  p->divCPB = make_fastdiv(static_cast<uint32_t>(mla::HEAD_DIM / 16 / s->head_dim_granularity));
  p->divG = make_fastdiv(static_cast<uint32_t>(p->G));
  p->divT = make_fastdiv(static_cast<uint32_t>(p->T));
  *rows = r;
  return MLA_OK;
}

// ---------------------------------------------------------------- Q tensor map
// cuTensorMapEncodeTiled comes from the driver through the runtime's entry-point query, so the
// library needs no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

mla_status_t get_encode_fn(EncodeTiledFn* fn) {
  static std::mutex mu;
  static EncodeTiledFn cached = nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!cached) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr);
    if (e != cudaSuccess || qr != cudaDriverEntryPointSuccess || !ptr)
      return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(e));
    cached = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  *fn = cached;
  return MLA_OK;
}

// q [B*T][H][576] bf16 as a 3-D tensor (dims innermost); one box = 64 dims x 64 heads of one query
// token, written in the 128-byte swizzle the MMA descriptors expect.  Heads past H read as zero.
mla_status_t make_q_map(CUtensorMap* map, const void* q, int H, int BT) {
  EncodeTiledFn enc = nullptr;
  mla_status_t st = get_encode_fn(&enc);
  if (st != MLA_OK) return st;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::HEAD_DIM), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(BT)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::HEAD_DIM) * 2,
                                 static_cast<cuuint64_t>(mla::HEAD_DIM) * 2 * static_cast<cuuint64_t>(H)};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(mla::HPC), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(q) failed (%d)", static_cast<int>(r));
  return MLA_OK;
}

unsigned int* status_ptr() {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), mla::g_status_word) != cudaSuccess) return nullptr;
  return p;
}

// Wait bound of the decode kernel's mbarrier waits, and the one-shot test hook.
void set_wait_params(mla::DecodeParams* p) {
  std::lock_guard<std::mutex> lk(g_mu);
  p->wait_limit_ns = g_wait_limit_ns;
  p->inject = g_inject_once;
  g_inject_once = mla::INJECT_NONE;
}

// The three launches of one decode call on `stream`: plan -> decode -> combine.  The decode and
// combine kernels are launched as programmatic dependents of the kernel before them, so their
// launch and (for the decode kernel) prologue overlap the previous kernel; each waits for its
// predecessor's results with griddepcontrol.wait.  With timing events set, the events bracket the
// decode launch (the event between plan and decode then serialises the two).
mla_status_t launch_path(const mla::DecodeParams& p, int NC, const uint32_t* cache_lengths, uint32_t max_cache_length,
                         cudaStream_t stream, bool timing, int mode = mla::SCALE_TOKEN) {
  mla::mla_plan_kernel<<<1, mla::PLAN_THREADS, 0, stream>>>(
      cache_lengths, p.B, p.T, p.G, max_cache_length, NC, const_cast<int32_t*>(p.item_start),
      const_cast<int32_t*>(p.item_nvis), const_cast<int32_t*>(p.cluster_first), const_cast<int32_t*>(p.hdr), p.status);
  MLA_CUDA(cudaGetLastError());

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * NC);
  cfg.blockDim = dim3(mla::NUM_THREADS);
  // block scales with g <= 9 take the kernel mode whose producer brings the own keys' block scales
  // into shared memory with the ring stage
  const bool block_ring = mode == mla::SCALE_TOKEN && p.SG > 1 && p.SG <= mla::BSC_MAX_G;
  const bool big_smem = mode == mla::SCALE_FOLD || mode == mla::SCALE_FP8PV || block_ring;
  cfg.dynamicSmemBytes = big_smem ? mla::SMEM_ALLOC_FOLD : mla::SMEM_ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (timing) MLA_CUDA(cudaEventRecord(g_ev_before, stream));
  if (mode == mla::SCALE_FOLD) {
    MLA_CUDA(cudaLaunchKernelEx(&cfg, mla::mla_decode_kernel<mla::SCALE_FOLD>, p));
  } else if (mode == mla::SCALE_FP8PV) {
    MLA_CUDA(cudaLaunchKernelEx(&cfg, mla::mla_decode_kernel<mla::SCALE_FP8PV>, p));
  } else if (block_ring) {
    MLA_CUDA(cudaLaunchKernelEx(&cfg, mla::mla_decode_kernel<mla::SCALE_BLOCKR>, p));
  } else if (p.SG > 1) {
    MLA_CUDA(cudaLaunchKernelEx(&cfg, mla::mla_decode_kernel<mla::SCALE_BLOCK>, p));
  } else {
    MLA_CUDA(cudaLaunchKernelEx(&cfg, mla::mla_decode_kernel<mla::SCALE_TOKEN>, p));
  }
  if (timing) MLA_CUDA(cudaEventRecord(g_ev_after, stream));

  const int per_item = mla::MROWS / mla::COMBINE_HEADS;
  const int64_t cgrid = static_cast<int64_t>(p.items) * per_item;
  if (cgrid > 0x7FFFFFFF) return fail(MLA_ERR_UNSUPPORTED, "combine grid too large");
  cudaLaunchConfig_t ccfg = {};
  ccfg.gridDim = dim3(static_cast<unsigned>(cgrid));
  ccfg.blockDim = dim3(32 * mla::COMBINE_HEADS);
  ccfg.dynamicSmemBytes = 0;
  ccfg.stream = stream;
  ccfg.attrs = &attr[1];
  ccfg.numAttrs = 1;
  MLA_CUDA(cudaLaunchKernelEx(&ccfg, mla::mla_combine_kernel, p));
  return MLA_OK;
}

}  // namespace

// ---------------------------------------------------------------- fixed scratch (no-allocation entry)
// Some callers cannot allocate device memory while they run (CUDA graph capture, allocators that own
// the whole device, real-time services that forbid allocation after start-up).  For them the decode
// also runs on one statically sized device array instead of the lazily allocated workspace.
namespace {

constexpr int kNoAllocMaxItems = 65536;      // (request, query token, head group) triples per call
constexpr int kNoAllocMaxClusters = 80;      // 2-CTA clusters the split is cut into (B200 default: 74)

constexpr size_t noalloc_up(size_t v) { return (v + 255) / 256 * 256; }
constexpr size_t kNoAllocBytes =
    noalloc_up(64) + noalloc_up(sizeof(int32_t) * (kNoAllocMaxItems + 1)) + noalloc_up(sizeof(int32_t) * kNoAllocMaxItems) +
    noalloc_up(sizeof(int32_t) * kNoAllocMaxClusters) + noalloc_up(sizeof(float) * 2 * kNoAllocMaxClusters * mla::MROWS) +
    noalloc_up(sizeof(float) * 2 * kNoAllocMaxClusters * mla::MROWS * mla::V_DIM);

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];

}  // namespace

// The scratch itself: about 42.5 MB of device memory on every GPU that loads this library, held
// until the process exits.  Host code must not pass this symbol to a kernel (in host code it names
// a host-side stand-in); it uses the device address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

// Device address of the scratch for the current device, looked up once per device.
mla_status_t noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(MLA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" {

const char* mla_version(void) { return "0.1.0"; }

const char* mla_last_error_string(void) { return g_last_error.c_str(); }

mla_status_t mla_set_num_clusters(int32_t num_clusters) {
  if (num_clusters < 0 || num_clusters > 65535) return fail(MLA_ERR_INVALID_ARG, "num_clusters out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  g_forced_nc = num_clusters;
  return MLA_OK;
}

mla_status_t mla_set_wait_limit_ns(uint64_t ns) {
  if (ns < 1000000ull || ns > 60000000000ull)
    return fail(MLA_ERR_INVALID_ARG, "wait limit %llu ns outside [1 ms, 60 s]", static_cast<unsigned long long>(ns));
  std::lock_guard<std::mutex> lk(g_mu);
  g_wait_limit_ns = ns;
  return MLA_OK;
}

mla_status_t mla_debug_withhold_arrival_once(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_inject_once = mla::INJECT_SKIP_Q_ARRIVAL;
  return MLA_OK;
}

mla_status_t mla_set_timing_events(cudaEvent_t before, cudaEvent_t after) {
  if ((before == nullptr) != (after == nullptr)) return fail(MLA_ERR_INVALID_ARG, "pass both events or neither");
  g_ev_before = before;
  g_ev_after = after;
  return MLA_OK;
}

int32_t mla_get_num_clusters(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return -1;
  int nc = 0;
  if (device_setup(dev, &nc) != MLA_OK) return -1;
  return nc;
}

}  // extern "C"

namespace {
// Body of mla_decode_paged_fp8, mla_decode_paged_fp8_scale_folded and mla_decode_paged_fp8_e4m3_pv
// (workspace from the pool).  mode: mla::SCALE_TOKEN (per-token or block scales by the shape),
// mla::SCALE_FOLD or mla::SCALE_FP8PV.
mla_status_t decode_alloc(const void* q, const void* blocks, const float* scales, const uint32_t* cache_lengths,
                          const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
                          uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx,
                          float softmax_scale, const mla_paged_shape_t* shape, void* out, float* lse,
                          cudaStream_t stream, int mode) {
  mla::DecodeParams p{};
  uint64_t rows = 0;
  mla_status_t st = check_cache(blocks, scales, cache_lengths, lookup_table, max_prompt_length, max_cache_length,
                                layer_idx, shape, &p, &rows);
  if (st != MLA_OK) return st;
  if (mode == mla::SCALE_FOLD && p.SG != 1)
    return fail(MLA_ERR_UNSUPPORTED, "the scale-folding decode takes one scale per token (head_dim_granularity 1)");
  if (mode == mla::SCALE_FP8PV && p.SG != 1)
    return fail(MLA_ERR_UNSUPPORTED, "the e4m3 P.V decode takes one scale per token (head_dim_granularity 1)");
  if (!q || !out) return fail(MLA_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(MLA_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale)) return fail(MLA_ERR_INVALID_ARG, "softmax_scale is NaN");
  if (p.B == 0) return MLA_OK;
  const int64_t items64 = static_cast<int64_t>(p.B) * p.T * p.G;
  if (items64 > (1 << 24)) return fail(MLA_ERR_UNSUPPORTED, "too many (request, token, head-group) items");
  p.items = static_cast<int>(items64);

  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index too large");
  int NC = 0;
  st = device_setup(dev, &NC);
  if (st != MLA_OK) return st;
  p.NC = NC;

  const WsLayout L = ws_layout(p.items, NC);
  void* ws = nullptr;
  st = ensure_workspace(dev, L.total, &ws);
  if (st != MLA_OK) return st;
  char* w = static_cast<char*>(ws);
  p.hdr = reinterpret_cast<int32_t*>(w + L.hdr);
  p.item_start = reinterpret_cast<int32_t*>(w + L.item_start);
  p.item_nvis = reinterpret_cast<int32_t*>(w + L.item_nvis);
  p.cluster_first = reinterpret_cast<int32_t*>(w + L.cluster_first);
  p.part_lse = reinterpret_cast<float*>(w + L.part_lse);
  p.part_o = reinterpret_cast<float*>(w + L.part_o);
  p.q = static_cast<const uint16_t*>(q);
  st = make_q_map(&p.tmap_q, q, p.H, p.B * p.T);
  if (st != MLA_OK) return st;
  p.slut = scales_lookup_table;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return fail(MLA_ERR_CUDA, "status word address unavailable");
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  set_wait_params(&p);
#ifdef MLA_TRACE
  p.trace = g_trace;
#endif

  return launch_path(p, NC, cache_lengths, max_cache_length, stream, g_ev_before && g_ev_after, mode);
}
}  // namespace

extern "C" {

mla_status_t mla_decode_paged_fp8(const void* q, const void* blocks, const float* scales,
                                  const uint32_t* cache_lengths, const uint32_t* lookup_table,
                                  const uint32_t* scales_lookup_table, uint32_t max_prompt_length,
                                  uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
                                  const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream) {
  return decode_alloc(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length,
                      max_cache_length, layer_idx, softmax_scale, shape, out, lse, stream, mla::SCALE_TOKEN);
}

mla_status_t mla_decode_paged_fp8_scale_folded(const void* q, const void* blocks, const float* scales,
                                               const uint32_t* cache_lengths, const uint32_t* lookup_table,
                                               const uint32_t* scales_lookup_table, uint32_t max_prompt_length,
                                               uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
                                               const mla_paged_shape_t* shape, void* out, float* lse,
                                               cudaStream_t stream) {
  return decode_alloc(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length,
                      max_cache_length, layer_idx, softmax_scale, shape, out, lse, stream, mla::SCALE_FOLD);
}

mla_status_t mla_decode_paged_fp8_e4m3_pv(const void* q, const void* blocks, const float* scales,
                                          const uint32_t* cache_lengths, const uint32_t* lookup_table,
                                          const uint32_t* scales_lookup_table, uint32_t max_prompt_length,
                                          uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
                                          const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream) {
  return decode_alloc(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length,
                      max_cache_length, layer_idx, softmax_scale, shape, out, lse, stream, mla::SCALE_FP8PV);
}

}  // extern "C"

namespace {
// ---------------------------------------------------------------- decode from host buffers
// Per device: a staging area in device memory for the call's inputs and outputs, two streams for
// the copies (host -> device, device -> host) and an event per chunk and direction.
constexpr int kMaxHostChunks = 16;
struct HostPipe {
  void* staging = nullptr;
  size_t bytes = 0;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_end = nullptr;
  cudaEvent_t ev_in[kMaxHostChunks] = {}, ev_dec[kMaxHostChunks] = {};
};
std::mutex g_hp_mu;
HostPipe g_hp[kMaxDevices];

mla_status_t host_pipe(int dev, size_t bytes, HostPipe** out) {
  HostPipe& h = g_hp[dev];
  if (!h.s_in) {
    MLA_CUDA(cudaStreamCreateWithFlags(&h.s_in, cudaStreamNonBlocking));
    MLA_CUDA(cudaStreamCreateWithFlags(&h.s_out, cudaStreamNonBlocking));
    MLA_CUDA(cudaEventCreateWithFlags(&h.ev_start, cudaEventDisableTiming));
    MLA_CUDA(cudaEventCreateWithFlags(&h.ev_end, cudaEventDisableTiming));
    for (int i = 0; i < kMaxHostChunks; ++i) {
      MLA_CUDA(cudaEventCreateWithFlags(&h.ev_in[i], cudaEventDisableTiming));
      MLA_CUDA(cudaEventCreateWithFlags(&h.ev_dec[i], cudaEventDisableTiming));
    }
  }
  if (h.bytes < bytes) {
    if (h.staging) {
      MLA_CUDA(cudaDeviceSynchronize());
      MLA_CUDA(cudaFree(h.staging));
      h.staging = nullptr;
      h.bytes = 0;
    }
    const size_t want = align_up(bytes + bytes / 8, 1 << 20);
    cudaError_t e = cudaMalloc(&h.staging, want);
    if (e != cudaSuccess) {
      h.staging = nullptr;
      return fail(MLA_ERR_WORKSPACE, "host-call staging cudaMalloc(%zu) failed: %s", want, cudaGetErrorString(e));
    }
    h.bytes = want;
  }
  *out = &h;
  return MLA_OK;
}

// Copies of a host range to device (or back) as one cudaMemcpyAsync each.
mla_status_t copy_async(void* dst, const void* src, size_t n, cudaMemcpyKind kind, cudaStream_t s) {
  if (n) MLA_CUDA(cudaMemcpyAsync(dst, src, n, kind, s));
  return MLA_OK;
}
}  // namespace

extern "C" {

mla_status_t mla_decode_paged_fp8_host(const void* q_host, const void* blocks, const float* scales,
                                       const uint32_t* cache_lengths_host, const uint32_t* lookup_table_host,
                                       const uint32_t* scales_lookup_table_host, uint32_t max_prompt_length,
                                       uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
                                       const mla_paged_shape_t* shape, void* out_host, float* lse_host,
                                       int32_t variant, int32_t num_chunks, cudaStream_t stream) {
  if (!shape) return fail(MLA_ERR_INVALID_ARG, "shape is NULL");
  if (!q_host || !cache_lengths_host || !lookup_table_host || !out_host)
    return fail(MLA_ERR_INVALID_ARG, "q_host, cache_lengths_host, lookup_table_host and out_host must be non-NULL");
  if (variant < MLA_VARIANT_DECODE || variant > MLA_VARIANT_E4M3_PV)
    return fail(MLA_ERR_INVALID_ARG, "variant %d is not one of MLA_VARIANT_*", variant);
  if (num_chunks < 0 || num_chunks > kMaxHostChunks)
    return fail(MLA_ERR_INVALID_ARG, "num_chunks %d outside [0, %d]", num_chunks, kMaxHostChunks);
  // the same checks as the device entry points, before anything is enqueued (stand-in device
  // pointers for the staged tables: only their presence is checked here)
  {
    mla::DecodeParams p{};
    uint64_t rows = 0;
    const mla_status_t st = check_cache(blocks, scales, cache_lengths_host, lookup_table_host, max_prompt_length,
                                        max_cache_length, layer_idx, shape, &p, &rows);
    if (st != MLA_OK) return st;
    if (variant != MLA_VARIANT_DECODE && p.SG != 1)
      return fail(MLA_ERR_UNSUPPORTED, "the scale-folding and e4m3 P.V decodes take one scale per token");
    if (!(softmax_scale == softmax_scale)) return fail(MLA_ERR_INVALID_ARG, "softmax_scale is NaN");
  }
  const int B = shape->batch;
  if (B == 0) return MLA_OK;
  const size_t T = max_prompt_length, H = static_cast<size_t>(shape->num_q_heads);
  const size_t MP = static_cast<size_t>(shape->max_pages);
  const size_t q_row = T * H * mla::HEAD_DIM * 2, o_row = T * H * mla::V_DIM * 2, l_row = T * H * 4;
  const size_t t_row = MP * 4;
  size_t o = 0;
  const size_t off_q = o;    o = align_up(o + q_row * B, 256);
  const size_t off_len = o;  o = align_up(o + 4 * static_cast<size_t>(B), 256);
  const size_t off_lut = o;  o = align_up(o + t_row * B, 256);
  const size_t off_slut = o; o = align_up(o + (scales_lookup_table_host ? t_row * B : 0), 256);
  const size_t off_out = o;  o = align_up(o + o_row * B, 256);
  const size_t off_lse = o;  o = align_up(o + l_row * B, 256);

  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lk(g_hp_mu);
  HostPipe* h = nullptr;
  mla_status_t st = host_pipe(dev, o, &h);
  if (st != MLA_OK) return st;
  char* d = static_cast<char*>(h->staging);
  const int nch = num_chunks > 0 ? (num_chunks < B ? num_chunks : B) : (B >= 64 ? 4 : B >= 16 ? 2 : 1);
  const int mode = variant == MLA_VARIANT_SCALE_FOLDED ? mla::SCALE_FOLD
                 : variant == MLA_VARIANT_E4M3_PV ? mla::SCALE_FP8PV : mla::SCALE_TOKEN;

  // Chunk i: host -> device copies on s_in, its decode on `stream`, device -> host copies on
  // s_out; copies of one chunk overlap the decode of another.  The staging area is reused by the
  // next call, whose first copy waits for everything this call enqueued on `stream` (ev_start).
  MLA_CUDA(cudaEventRecord(h->ev_start, stream));
  MLA_CUDA(cudaStreamWaitEvent(h->s_in, h->ev_start, 0));
  MLA_CUDA(cudaStreamWaitEvent(h->s_out, h->ev_start, 0));
  mla_paged_shape_t cs = *shape;
  for (int i = 0; i < nch && st == MLA_OK; ++i) {
    const size_t b0 = static_cast<size_t>(B) * i / nch, b1 = static_cast<size_t>(B) * (i + 1) / nch, nb = b1 - b0;
    const char* hq = static_cast<const char*>(q_host);
    if ((st = copy_async(d + off_q + q_row * b0, hq + q_row * b0, q_row * nb, cudaMemcpyHostToDevice, h->s_in)) ||
        (st = copy_async(d + off_len + 4 * b0, cache_lengths_host + b0, 4 * nb, cudaMemcpyHostToDevice, h->s_in)) ||
        (st = copy_async(d + off_lut + t_row * b0, lookup_table_host + MP * b0, t_row * nb, cudaMemcpyHostToDevice,
                         h->s_in)))
      break;
    if (scales_lookup_table_host &&
        (st = copy_async(d + off_slut + t_row * b0, scales_lookup_table_host + MP * b0, t_row * nb,
                         cudaMemcpyHostToDevice, h->s_in)))
      break;
    if (cudaEventRecord(h->ev_in[i], h->s_in) != cudaSuccess || cudaStreamWaitEvent(stream, h->ev_in[i], 0) != cudaSuccess) {
      st = fail(MLA_ERR_CUDA, "event record / wait failed");
      break;
    }
    cs.batch = static_cast<int32_t>(nb);
    st = decode_alloc(d + off_q + q_row * b0, blocks, scales, reinterpret_cast<const uint32_t*>(d + off_len) + b0,
                      reinterpret_cast<const uint32_t*>(d + off_lut) + MP * b0,
                      scales_lookup_table_host ? reinterpret_cast<const uint32_t*>(d + off_slut) + MP * b0 : nullptr,
                      max_prompt_length, max_cache_length, layer_idx, softmax_scale, &cs, d + off_out + o_row * b0,
                      lse_host ? reinterpret_cast<float*>(d + off_lse + l_row * b0) : nullptr, stream, mode);
    if (st != MLA_OK) break;
    if (cudaEventRecord(h->ev_dec[i], stream) != cudaSuccess || cudaStreamWaitEvent(h->s_out, h->ev_dec[i], 0) != cudaSuccess) {
      st = fail(MLA_ERR_CUDA, "event record / wait failed");
      break;
    }
    if ((st = copy_async(static_cast<char*>(out_host) + o_row * b0, d + off_out + o_row * b0, o_row * nb,
                         cudaMemcpyDeviceToHost, h->s_out)))
      break;
    if (lse_host && (st = copy_async(reinterpret_cast<char*>(lse_host) + l_row * b0, d + off_lse + l_row * b0,
                                     l_row * nb, cudaMemcpyDeviceToHost, h->s_out)))
      break;
  }
  if (st != MLA_OK) {
    // nothing enqueued by this call may still touch the caller's host buffers when it returns
    cudaStreamSynchronize(h->s_in);
    cudaStreamSynchronize(stream);
    cudaStreamSynchronize(h->s_out);
    return st;
  }
  MLA_CUDA(cudaEventRecord(h->ev_end, h->s_out));
  MLA_CUDA(cudaStreamWaitEvent(stream, h->ev_end, 0));
  return MLA_OK;
}

mla_status_t mla_gather_dequant_bf16(const void* blocks, const float* scales, const uint32_t* cache_lengths,
                                     const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
                                     uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx,
                                     const mla_paged_shape_t* shape, void* out_k, uint32_t max_keys,
                                     cudaStream_t stream) {
  mla::DecodeParams p{};
  uint64_t rows = 0;
  mla_status_t st = check_cache(blocks, scales, cache_lengths, lookup_table, max_prompt_length, max_cache_length,
                                layer_idx, shape, &p, &rows);
  if (st != MLA_OK) return st;
  if (!out_k || !aligned16(out_k)) return fail(MLA_ERR_INVALID_ARG, "out_k must be non-NULL and 16-byte aligned");
  if (static_cast<uint64_t>(max_keys) < static_cast<uint64_t>(max_cache_length) + max_prompt_length)
    return fail(MLA_ERR_INVALID_ARG, "max_keys %u < max_cache_length + max_prompt_length", max_keys);
  if (p.B == 0) return MLA_OK;
  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index too large");
  int NC = 0;
  st = device_setup(dev, &NC);
  if (st != MLA_OK) return st;
  p.slut = scales_lookup_table;
  p.status = status_ptr();
  if (!p.status) return fail(MLA_ERR_CUDA, "status word address unavailable");
  p.wait_limit_ns = g_wait_limit_ns;
  const int tiles = static_cast<int>((static_cast<uint64_t>(max_keys) + mla::BN - 1) / mla::BN);
  const int64_t gx = static_cast<int64_t>(p.B) * tiles;
  if (gx > 0x7FFFFFFF) return fail(MLA_ERR_UNSUPPORTED, "grid too large");
  if (p.SG > 1) {
    mla::mla_dequant_kernel<true><<<dim3(static_cast<unsigned>(gx), 2), mla::DQ_THREADS, mla::DQ_SMEM_ALLOC, stream>>>(
        p, cache_lengths, static_cast<int>(max_keys), tiles, static_cast<uint16_t*>(out_k));
  } else {
    mla::mla_dequant_kernel<false><<<dim3(static_cast<unsigned>(gx), 2), mla::DQ_THREADS, mla::DQ_SMEM_ALLOC, stream>>>(
        p, cache_lengths, static_cast<int>(max_keys), tiles, static_cast<uint16_t*>(out_k));
  }
  MLA_CUDA(cudaGetLastError());
  return MLA_OK;
}

mla_status_t mla_kv_store_fp8(const void* latent, const uint32_t* cache_lengths, const uint32_t* lookup_table,
                              const uint32_t* scales_lookup_table, uint32_t num_new_tokens, uint32_t layer_idx,
                              const mla_paged_shape_t* s, void* blocks, float* scales, cudaStream_t stream) {
  if (!s) return fail(MLA_ERR_INVALID_ARG, "shape is NULL");
  if (!latent || !cache_lengths || !lookup_table || !blocks || !scales)
    return fail(MLA_ERR_INVALID_ARG, "latent, cache_lengths, lookup_table, blocks and scales must be non-NULL");
  if (s->batch < 0 || s->num_blocks < 1 || s->kv_dim < 1 || s->num_layers < 1 || s->page_size < 1 ||
      s->num_kv_heads < 1 || s->num_scale_blocks < 1 || s->head_dim_granularity < 1 || s->max_pages < 1)
    return fail(MLA_ERR_INVALID_ARG, "non-positive dimension in shape");
  if (s->head_dim != mla::HEAD_DIM) return fail(MLA_ERR_UNSUPPORTED, "head_dim must be 576 (got %d)", s->head_dim);
  if (s->num_kv_heads != 1) return fail(MLA_ERR_UNSUPPORTED, "num_kv_heads must be 1 (MLA latent cache)");
  if (s->head_dim_granularity != 1)
    return fail(MLA_ERR_UNSUPPORTED, "only one scale per token (head_dim_granularity 1) is implemented");
  if (layer_idx >= static_cast<uint32_t>(s->num_layers))
    return fail(MLA_ERR_INVALID_ARG, "layer_idx %u >= num_layers %d", layer_idx, s->num_layers);
  if (!aligned16(latent) || !aligned16(blocks) || !aligned16(scales))
    return fail(MLA_ERR_INVALID_ARG, "latent, blocks and scales must be 16-byte aligned");
  const uint64_t r = static_cast<uint64_t>(s->num_blocks) * s->kv_dim * s->num_layers * s->page_size;
  const uint64_t sr = static_cast<uint64_t>(s->num_scale_blocks) * s->kv_dim * s->num_layers * s->page_size;
  if (r >= (1ull << 40) || sr >= (1ull << 40)) return fail(MLA_ERR_UNSUPPORTED, "block pool too large");
  const uint64_t tokens = static_cast<uint64_t>(s->batch) * num_new_tokens;
  if (tokens == 0) return MLA_OK;
  if (tokens >= (1ull << 31)) return fail(MLA_ERR_UNSUPPORTED, "too many new tokens (%llu)", static_cast<unsigned long long>(tokens));
  mla::KvStoreParams p{};
  p.latent = static_cast<const uint16_t*>(latent);
  p.cache_lengths = cache_lengths;
  p.lut = lookup_table;
  p.slut = scales_lookup_table;
  p.blocks = static_cast<uint8_t*>(blocks);
  p.scales = scales;
  p.status = status_ptr();
  if (!p.status) return fail(MLA_ERR_CUDA, "status word address unavailable");
  p.B = s->batch;
  p.T = static_cast<int>(num_new_tokens);
  p.P = s->page_size;
  p.KVD = s->kv_dim;
  p.NL = s->num_layers;
  p.layer = static_cast<int>(layer_idx);
  p.NB = s->num_blocks;
  p.NSB = s->num_scale_blocks;
  p.max_pages = s->max_pages;
  p.divT = make_fastdiv(num_new_tokens);
  const uint64_t per_cta = 32 * mla::KVS_WARPS / mla::KVS_LANES;     // tokens per CTA
  const uint64_t grid = (tokens + per_cta - 1) / per_cta;
  mla::mla_kv_store_kernel<<<static_cast<unsigned>(grid), 32 * mla::KVS_WARPS, 0, stream>>>(p);
  MLA_CUDA(cudaGetLastError());
  return MLA_OK;
}

#ifdef MLA_TRACE
// Trace builds only: cluster 0 of later decodes writes per-stage %clock64 stamps to `buf`
// (2 * TRACE_TILES * TRACE_EVENTS uint64 values).
mla_status_t mla_debug_set_trace(unsigned long long* buf) {
  g_trace = buf;
  return MLA_OK;
}

// Trace builds only: copies the %globaltimer marks of the last decode call (plan end, first decode
// CTA entry, last decode CTA exit, first combine CTA past its wait, last combine warp done, first
// combine CTA entry) to out8 and, if reset, re-arms them.
mla_status_t mla_debug_marks(unsigned long long* out8, int reset) {
  MLA_CUDA(cudaDeviceSynchronize());
  MLA_CUDA(cudaMemcpyFromSymbol(out8, mla::g_trace_marks, 8 * sizeof(unsigned long long)));
  if (reset) {
    const unsigned long long init[8] = {0ull, ~0ull, 0ull, ~0ull, 0ull, ~0ull, 0ull, 0ull};
    MLA_CUDA(cudaMemcpyToSymbol(mla::g_trace_marks, init, sizeof(init)));
  }
  return MLA_OK;
}
#endif

// Same decode as mla_decode_paged_fp8, but on the fixed scratch: no device memory is allocated or
// freed.  The first call on a device looks up the scratch address (and, like the regular entry,
// sets the kernels' shared-memory attribute); make that first call before any stream capture.
// Calls share the scratch, so two calls that overlap on the GPU (different streams or devices'
// worth of work racing on one device) corrupt each other; serialise them.  Nothing in the scratch
// has to start at zero: every call writes what it reads.
mla_status_t mla_decode_paged_fp8_noalloc(const void* q, const void* blocks, const float* scales,
                                          const uint32_t* cache_lengths, const uint32_t* lookup_table,
                                          const uint32_t* scales_lookup_table, uint32_t max_prompt_length,
                                          uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
                                          const mla_paged_shape_t* shape, void* out, float* lse,
                                          cudaStream_t stream) {
  mla::DecodeParams p{};
  uint64_t rows = 0;
  mla_status_t st = check_cache(blocks, scales, cache_lengths, lookup_table, max_prompt_length, max_cache_length,
                                layer_idx, shape, &p, &rows);
  if (st != MLA_OK) return st;
  if (!q || !out) return fail(MLA_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(MLA_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale)) return fail(MLA_ERR_INVALID_ARG, "softmax_scale is NaN");
  if (p.B == 0) return MLA_OK;
  const int64_t items64 = static_cast<int64_t>(p.B) * p.T * p.G;
  if (items64 > kNoAllocMaxItems)
    return fail(MLA_ERR_UNSUPPORTED,
                "batch * max_prompt_length * ceil(num_q_heads / 128) = %lld exceeds the fixed scratch limit of %d",
                static_cast<long long>(items64), kNoAllocMaxItems);
  p.items = static_cast<int>(items64);

  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index too large");
  int NC = 0;
  st = device_setup(dev, &NC);
  if (st != MLA_OK) return st;
  if (NC > kNoAllocMaxClusters)
    return fail(MLA_ERR_UNSUPPORTED,
                "the no-allocation decode splits the keys over at most %d clusters, this call would use %d "
                "(lower it with mla_set_num_clusters)", kNoAllocMaxClusters, NC);
  p.NC = NC;

  void* ws = nullptr;
  st = noalloc_scratch(dev, &ws);
  if (st != MLA_OK) return st;
  const WsLayout L = ws_layout(p.items, NC);
  if (L.total > kNoAllocBytes) return fail(MLA_ERR_UNSUPPORTED, "problem needs more than the fixed scratch");
  char* w = static_cast<char*>(ws);
  p.hdr = reinterpret_cast<int32_t*>(w + L.hdr);
  p.item_start = reinterpret_cast<int32_t*>(w + L.item_start);
  p.item_nvis = reinterpret_cast<int32_t*>(w + L.item_nvis);
  p.cluster_first = reinterpret_cast<int32_t*>(w + L.cluster_first);
  p.part_lse = reinterpret_cast<float*>(w + L.part_lse);
  p.part_o = reinterpret_cast<float*>(w + L.part_o);
  p.q = static_cast<const uint16_t*>(q);
  st = make_q_map(&p.tmap_q, q, p.H, p.B * p.T);
  if (st != MLA_OK) return st;
  p.slut = scales_lookup_table;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return fail(MLA_ERR_CUDA, "status word address unavailable");
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  set_wait_params(&p);

  return launch_path(p, NC, cache_lengths, max_cache_length, stream, false);
}

mla_status_t mla_merge_lse_parts_bf16(const void* outs, const float* lses, int32_t num_parts, int64_t rows,
                                      void* out, float* lse, cudaStream_t stream) {
  if (num_parts < 1 || rows < 0) return fail(MLA_ERR_INVALID_ARG, "num_parts must be >= 1 and rows >= 0");
  if (rows == 0) return MLA_OK;
  if (!outs || !lses || !out) return fail(MLA_ERR_INVALID_ARG, "outs, lses and out must be non-NULL");
  if (!aligned16(outs) || !aligned16(out)) return fail(MLA_ERR_INVALID_ARG, "outs and out must be 16-byte aligned");
  if (rows > (1ll << 40) / num_parts) return fail(MLA_ERR_UNSUPPORTED, "too many rows");
  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  int sms = 0;
  MLA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  long long blocks = (rows + mla::MERGE_WARPS - 1) / mla::MERGE_WARPS;
  if (blocks > 8ll * sms) blocks = 8ll * sms;
  mla::mla_merge_parts_kernel<<<static_cast<unsigned>(blocks), 32 * mla::MERGE_WARPS, 0, stream>>>(
      static_cast<const uint16_t*>(outs), lses, num_parts, static_cast<long long>(rows), static_cast<uint16_t*>(out), lse);
  MLA_CUDA(cudaGetLastError());
  return MLA_OK;
}

mla_status_t mla_get_device_status(cudaStream_t stream) {
  MLA_CUDA(cudaStreamSynchronize(stream));
  unsigned int v = 0, zero = 0;
  MLA_CUDA(cudaMemcpyFromSymbol(&v, mla::g_status_word, sizeof(v)));
  MLA_CUDA(cudaMemcpyToSymbol(mla::g_status_word, &zero, sizeof(zero)));
  if (v & mla::STATUS_TIMEOUT) return fail(MLA_ERR_TIMEOUT, "a kernel wait timed out (status 0x%x)", v);
  if (v & mla::STATUS_BOUNDS) return fail(MLA_ERR_DEVICE_BOUNDS, "page id or cache length out of range (status 0x%x)", v);
  if (v & mla::STATUS_LAYOUT)
    return fail(MLA_ERR_UNSUPPORTED,
                "dynamic shared memory base not aligned as the scale-folding and e4m3 P.V decodes need (status 0x%x)", v);
  return MLA_OK;
}

mla_status_t mla_release_workspace(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (int d = 0; d < kMaxDevices; ++d) {
    if (!g_ws[d].ptr) continue;
    MLA_CUDA(cudaSetDevice(d));
    MLA_CUDA(cudaDeviceSynchronize());
    MLA_CUDA(cudaFree(g_ws[d].ptr));
    g_ws[d].ptr = nullptr;
    g_ws[d].bytes = 0;
  }
  cudaSetDevice(cur);
  return MLA_OK;
}

}  // extern "C"
