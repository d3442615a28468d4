// gmla.cu — the C ABI declared in include/gmla.h: argument checks, workspace
// layout, tensor-map construction and kernel dispatch. Every compute step runs
// in the kernels of gemm_tc.cu, decode_tc.cu, prefill_tc.cu (bf16, tcgen05) or
// simt_f32.cu (fp32, CUDA cores); there is no host fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/gmla.h"
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

using namespace gmla;

namespace {

thread_local std::string g_err;

gmla_status fail(gmla_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
gmla_status fail(gmla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

gmla_status cuda_fail(cudaError_t e, const char* where) {
  return fail(GMLA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// tensor maps through the driver entry point (the library does not link libcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

const char* status_str(gmla_status s) {
  switch (s) {
    case GMLA_OK: return "ok";
    case GMLA_ERR_INVALID_ARG: return "invalid argument";
    case GMLA_ERR_UNSUPPORTED: return "unsupported shape or mode (no fallback path exists)";
    case GMLA_ERR_WORKSPACE: return "workspace missing or too small";
    case GMLA_ERR_CUDA: return "CUDA error";
    case GMLA_ERR_TIMEOUT: return "a device-side wait timed out";
    case GMLA_ERR_DEVICE_RANGE: return "a kernel saw an out-of-range sequence length or page";
  }
  return "unknown status";
}

gmla_status check_cfg(const gmla_config* c) {
  if (!c) return fail(GMLA_ERR_INVALID_ARG, "config is NULL");
  if (c->d_model <= 0 || c->n_heads <= 0 || c->d_h <= 0 || c->d_c <= 0 || c->d_rope < 0 || c->d_cq < 0)
    return fail(GMLA_ERR_INVALID_ARG, "non-positive dimension in config");
  if (c->d_rope % 2) return fail(GMLA_ERR_INVALID_ARG, "d_rope must be even (RoPE rotates pairs)");
  if (c->gate_mode < GMLA_GATE_CHANNEL || c->gate_mode > GMLA_GATE_HEAD_TERNARY)
    return fail(GMLA_ERR_INVALID_ARG, "gate_mode must be one of the gmla_gate_mode values");
  if (c->gate_mode == GMLA_GATE_HEAD_TOPK && (c->gate_topk < 1 || c->gate_topk > c->n_heads))
    return fail(GMLA_ERR_INVALID_ARG, "gate_topk must be in [1, n_heads] for GMLA_GATE_HEAD_TOPK");
  if (c->cache_dtype != GMLA_CACHE_SAME && c->cache_dtype != GMLA_CACHE_FP8_E4M3)
    return fail(GMLA_ERR_INVALID_ARG, "cache_dtype must be a gmla_cache_dtype value");
  if (c->cache_dtype == GMLA_CACHE_FP8_E4M3 &&
      (c->dtype != GMLA_BF16 || !(c->cache_scale > 0.f) || !std::isfinite(c->cache_scale)))
    return fail(GMLA_ERR_INVALID_ARG, "an FP8 cache needs the bf16 dtype and a finite cache_scale > 0");
  if (c->dtype != GMLA_BF16 && c->dtype != GMLA_FP32) return fail(GMLA_ERR_INVALID_ARG, "dtype");
  if (!(c->softmax_scale > 0.f) || !std::isfinite(c->softmax_scale))
    return fail(GMLA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (c->d_rope && !(c->rope_base > 1.f)) return fail(GMLA_ERR_INVALID_ARG, "rope_base must be > 1");
  return GMLA_OK;
}

// The same checks as check_cfg, without touching the thread's last error (for
// the size queries, which return a status-free value).
bool cfg_valid(const gmla_config* c) {
  if (!c) return false;
  if (c->d_model <= 0 || c->n_heads <= 0 || c->d_h <= 0 || c->d_c <= 0 || c->d_rope < 0 || c->d_cq < 0)
    return false;
  if (c->d_rope % 2) return false;
  if (c->gate_mode < GMLA_GATE_CHANNEL || c->gate_mode > GMLA_GATE_HEAD_TERNARY) return false;
  if (c->gate_mode == GMLA_GATE_HEAD_TOPK && (c->gate_topk < 1 || c->gate_topk > c->n_heads)) return false;
  if (c->cache_dtype != GMLA_CACHE_SAME && c->cache_dtype != GMLA_CACHE_FP8_E4M3) return false;
  if (c->cache_dtype == GMLA_CACHE_FP8_E4M3 &&
      (c->dtype != GMLA_BF16 || !(c->cache_scale > 0.f) || !std::isfinite(c->cache_scale)))
    return false;
  if (c->dtype != GMLA_BF16 && c->dtype != GMLA_FP32) return false;
  if (!(c->softmax_scale > 0.f) || !std::isfinite(c->softmax_scale)) return false;
  if (c->d_rope && !(c->rope_base > 1.f)) return false;
  return true;
}

gmla_status check_ptr(const void* p, const char* name, bool required = true) {
  if (!p) return required ? fail(GMLA_ERR_INVALID_ARG, "%s is NULL", name) : GMLA_OK;
  if (!aligned16(p)) return fail(GMLA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return GMLA_OK;
}

#define GMLA_TRY(x)                         \
  do {                                      \
    gmla_status _s = (x);                   \
    if (_s != GMLA_OK) return _s;           \
  } while (0)

gmla_status check_cache(const gmla_config* c, const gmla_cache* k) {
  if (!k) return fail(GMLA_ERR_INVALID_ARG, "cache is NULL");
  GMLA_TRY(check_ptr(k->data, "cache.data"));
  if (k->batch <= 0) return fail(GMLA_ERR_INVALID_ARG, "cache.batch must be > 0");
  if (!k->paged) {
    if (k->capacity <= 0) return fail(GMLA_ERR_INVALID_ARG, "cache.capacity must be > 0");
  } else {
    GMLA_TRY(check_ptr(k->block_table, "cache.block_table"));
    if (k->page_size <= 0 || k->num_pages <= 0 || k->max_pages_per_seq <= 0)
      return fail(GMLA_ERR_INVALID_ARG, "paged cache sizes must be > 0");
    const int ps = k->page_size;
    const bool ok = (ps < 128) ? (ps >= 8 && (128 % ps) == 0) : (ps % 128 == 0);
    if (!ok) return fail(GMLA_ERR_UNSUPPORTED, "page_size %d: must divide 128 (>= 8) or be a multiple of 128", ps);
  }
  (void)c;
  return GMLA_OK;
}

CacheView cache_view(const gmla_config* c, const gmla_cache* k) {
  CacheView v{};
  v.data = k->data;
  v.block_table = k->block_table;
  v.paged = k->paged;
  v.batch = k->batch;
  v.capacity = k->capacity;
  v.page_size = k->page_size;
  v.num_pages = k->num_pages;
  v.max_pages_per_seq = k->max_pages_per_seq;
  v.row = c->d_c + c->d_rope;
  return v;
}

int gate_width(const gmla_config* c) {
  return c->gate_mode == GMLA_GATE_CHANNEL ? c->n_heads * c->d_h : c->n_heads;
}

// Most heads one decode query attends with: k under top-k gates (the others
// are skipped), else H. The attention kernel's head groups cover this many.
int decode_eff_heads(const gmla_config* c) {
  return c->gate_mode == GMLA_GATE_HEAD_TOPK ? c->gate_topk : c->n_heads;
}

EpiSeg plain_seg(void* out, int64_t row_stride, int block, int block_stride, int col_offset, bool f32,
                 const float* bias, bool rope, bool scatter) {
  EpiSeg e{};
  e.out = out;
  e.bias = bias;
  e.row_stride = row_stride;
  e.block = block;
  e.block_stride = block_stride;
  e.col_offset = col_offset;
  e.out_f32 = f32 ? 1 : 0;
  e.rope = rope ? 1 : 0;
  e.cache_scatter = scatter ? 1 : 0;
  return e;
}

// per-launch timing records
struct ProfRec {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
size_t g_prof_used = 0;
bool g_prof_open = false;
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_test_stall{0};   // armed by gmla_test_stall_next_decode

}  // namespace

namespace gmla {

void set_last_error(const char* msg) { g_err = msg ? msg : ""; }

int check_config(const ::gmla_config* c) { return check_cfg(c); }

void prof_begin(cudaStream_t st, const char* name) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_used == g_prof.size()) {
    ProfRec r{};
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return;
    g_prof.push_back(r);
  }
  g_prof[g_prof_used].name = name;
  cudaEventRecordWithFlags(g_prof[g_prof_used].start, st, cudaEventRecordExternal);
  g_prof_open = true;
}

void prof_end(cudaStream_t st) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_open) return;
  cudaEventRecordWithFlags(g_prof[g_prof_used].stop, st, cudaEventRecordExternal);
  ++g_prof_used;
  g_prof_open = false;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box_inner, uint32_t box1, uint32_t box2,
                  bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box_inner, box1, box2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                     uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t d1, uint64_t d2,
                     uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box_inner, uint32_t box1,
                     uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box_inner, box1, box2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gmla

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* gmla_status_string(gmla_status s) { return status_str(s); }
const char* gmla_last_error(void) { return g_err.c_str(); }
const char* gmla_version(void) { return "gmla 0.1.0 sm_100a"; }

uint64_t gmla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

gmla_status gmla_test_stall_next_decode(int32_t enable) {
  g_test_stall.store(enable ? 1 : 0);
  return GMLA_OK;
}

gmla_status gmla_profile_enable(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = enable != 0;
  g_prof_used = 0;
  g_prof_open = false;
  return GMLA_OK;
}

int32_t gmla_profile_count(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return static_cast<int32_t>(g_prof_used);
}

gmla_status gmla_profile_get(int32_t i, const char** name, float* ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (i < 0 || static_cast<size_t>(i) >= g_prof_used || !name || !ms)
    return fail(GMLA_ERR_INVALID_ARG, "profile record %d out of range", i);
  cudaError_t e = cudaEventSynchronize(g_prof[i].stop);
  if (e != cudaSuccess) return cuda_fail(e, "gmla_profile_get");
  e = cudaEventElapsedTime(ms, g_prof[i].start, g_prof[i].stop);
  if (e != cudaSuccess) return cuda_fail(e, "gmla_profile_get");
  *name = g_prof[i].name;
  return GMLA_OK;
}

// Bytes of the compressed query c^Q [T, d_cq] kept in the workspace (after the status word).
static size_t cq_bytes(const gmla_config* c, int32_t T) {
  if (c->d_cq <= 0) return 0;
  return align256(static_cast<size_t>(T) * c->d_cq * (c->dtype == GMLA_FP32 ? 4 : 2));
}

size_t gmla_latent_project_workspace_size(const gmla_config* cfg, int32_t T) {
  if (!cfg_valid(cfg) || T < 0) return 256;
  return 256 + cq_bytes(cfg, T);
}

size_t gmla_gate_out_workspace_size(const gmla_config* cfg, int32_t T) {
  if (!cfg_valid(cfg) || T < 0) return 256;
  const size_t es = cfg->dtype == GMLA_FP32 ? 4 : 2;
  size_t n = 256 + align256(static_cast<size_t>(T) * cfg->n_heads * cfg->d_h * es);
  if (cfg->dtype != GMLA_FP32 && T <= 256)
    n += gemm_swap_plan((cfg->d_model + 127) / 128, T, cfg->n_heads * cfg->d_h, num_sms()).ws_bytes;
  return n;
}

size_t gmla_decode_workspace_size(const gmla_config* cfg, int32_t B) {
  if (!cfg_valid(cfg) || B < 0) return 256;
  if (cfg->dtype == GMLA_FP32) return 256;
  return decode_layout(B, cfg->n_heads, decode_eff_heads(cfg), cfg->d_h, cfg->d_c, cfg->d_rope, num_sms(),
                       cfg->cache_dtype == GMLA_CACHE_FP8_E4M3).total;
}

size_t gmla_prefill_workspace_size(const gmla_config* cfg, int32_t T, int32_t B) {
  if (!cfg_valid(cfg) || T < 0 || B < 0) return 256;
  const size_t es = cfg->dtype == GMLA_FP32 ? 4 : 2;
  const size_t kv = static_cast<size_t>(T) * cfg->n_heads * cfg->d_h * es;
  return 256 + 2 * align256(kv);
}

gmla_status gmla_clear_status(void* workspace, void* stream) {
  if (!workspace) return fail(GMLA_ERR_WORKSPACE, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "gmla_clear_status");
}

gmla_status gmla_sync_status(const void* workspace, void* stream) {
  if (!workspace) return fail(GMLA_ERR_WORKSPACE, "workspace is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gmla_sync_status: stream");
  int v = 0;
  e = cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "gmla_sync_status: read");
  if (v == kStatusTimeout) return fail(GMLA_ERR_TIMEOUT, "a device-side wait timed out");
  if (v == kStatusRange) return fail(GMLA_ERR_DEVICE_RANGE, "a kernel saw an out-of-range length or page");
  return v == 0 ? GMLA_OK : fail(GMLA_ERR_CUDA, "unknown device status %d", v);
}

// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

struct ProjSeg {
  const void* W;
  int rows;
  EpiSeg e;
};

// One projection GEMM: act [T, K] times the weight segments, each segment with
// its own epilogue (tcgen05 kernel for bf16, CUDA-core kernel for fp32).
gmla_status project_gemm(const gmla_config* cfg, const void* act, int T, int K, const ProjSeg* segs, int ns,
                         const int32_t* positions, const int32_t* seq_ids, const CacheView& cv, int* status,
                         cudaStream_t st, const char* name) {
  const bool f32 = cfg->dtype == GMLA_FP32;
  const double log2_base = cfg->d_rope ? std::log2(static_cast<double>(cfg->rope_base)) : 0.0;
  if (f32) {
    F32Args a{};
    a.x = static_cast<const float*>(act);
    a.T = T;
    a.K = K;
    a.n_seg = ns;
    for (int i = 0; i < ns; ++i) {
      a.W[i] = static_cast<const float*>(segs[i].W);
      a.epi[i] = segs[i].e;
      a.seg_rows[i] = segs[i].rows;
    }
    a.positions = positions;
    a.seq_ids = seq_ids;
    a.cache = cv;
    a.log2_rope_base = log2_base;
    a.status = status;
    cudaError_t e = launch_gemm_f32(a, st);
    return e == cudaSuccess ? GMLA_OK : cuda_fail(e, name);
  }
  if (K % 8) return fail(GMLA_ERR_UNSUPPORTED, "%s: the bf16 path needs an inner dimension %% 8 == 0", name);
  int wtiles = 0;
  for (int i = 0; i < ns; ++i) wtiles += (segs[i].rows + 127) / 128;
  GemmArgs a{};
  const bool swap = T <= 256;
  const SwapPlan sp = gemm_swap_plan(wtiles, T, K, num_sms());
  const int bn = swap ? sp.bn : 256;
  const int wtile = gemm_weight_tile(swap, bn);
  if (!make_tmap_2d(&a.act, act, K, T, static_cast<uint64_t>(K) * 2, 64, swap ? bn : 128, true))
    return fail(GMLA_ERR_CUDA, "%s: tensor map for the activations failed", name);
  a.seg_tile_begin[0] = 0;
  for (int i = 0; i < ns; ++i) {
    if (!make_tmap_2d(&a.wt[i], segs[i].W, K, segs[i].rows, static_cast<uint64_t>(K) * 2, 64, wtile, true))
      return fail(GMLA_ERR_CUDA, "%s: tensor map for weight segment %d failed", name, i);
    a.epi[i] = segs[i].e;
    a.seg_rows[i] = segs[i].rows;
    a.seg_tile_begin[i + 1] = a.seg_tile_begin[i] + (segs[i].rows + wtile - 1) / wtile;
  }
  a.n_seg = ns;
  a.T = T;
  a.K = K;
  a.row_mode = 0;
  a.positions = positions;
  a.seq_ids = seq_ids;
  a.cache = cv;
  a.log2_rope_base = log2_base;
  a.status = status;
  if (swap) {
    a.splits = sp.splits;
    a.kb_per_split = sp.kb_per_split;
  }
  const int ttiles = swap ? sp.ttiles : (T + 127) / 128;
  cudaError_t e = launch_gemm_bf16(a, swap, bn, ttiles, st, name);
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, name);
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
gmla_status gmla_latent_project(const gmla_config* cfg, const gmla_weights* w, const void* x, int32_t T,
                                const int32_t* positions, const int32_t* seq_ids, const gmla_cache* cache,
                                void* q_out, float* gate_logits, void* workspace, size_t workspace_bytes,
                                void* stream) {
  GMLA_TRY(check_cfg(cfg));
  if (!w) return fail(GMLA_ERR_INVALID_ARG, "weights is NULL");
  if (T < 0) return fail(GMLA_ERR_INVALID_ARG, "T < 0");
  GMLA_TRY(check_cache(cfg, cache));
  if (!workspace || workspace_bytes < gmla_latent_project_workspace_size(cfg, T))
    return fail(GMLA_ERR_WORKSPACE, "latent_project needs %zu workspace bytes",
                gmla_latent_project_workspace_size(cfg, T));
  GMLA_TRY(check_ptr(workspace, "workspace"));
  if (T == 0) return GMLA_OK;
  const bool compressed = cfg->d_cq > 0;
  GMLA_TRY(check_ptr(x, "x"));
  GMLA_TRY(check_ptr(positions, "positions"));
  GMLA_TRY(check_ptr(seq_ids, "seq_ids"));
  GMLA_TRY(check_ptr(q_out, "q_out"));
  GMLA_TRY(check_ptr(gate_logits, "gate_logits"));
  GMLA_TRY(check_ptr(w->W_c, "W_c"));
  if (compressed) {
    GMLA_TRY(check_ptr(w->W_dq, "W_dq"));
    GMLA_TRY(check_ptr(w->W_uq, "W_uq"));
  } else {
    GMLA_TRY(check_ptr(w->W_q, "W_q"));
  }
  GMLA_TRY(check_ptr(w->W_g, "W_g"));
  if (cfg->d_rope) {
    GMLA_TRY(check_ptr(w->W_kr, "W_kr"));
    GMLA_TRY(check_ptr(w->W_qr, "W_qr"));
  }
  if (cfg->gate_bias) GMLA_TRY(check_ptr(w->b_g, "b_g"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = cfg->n_heads, dh = cfg->d_h, dc = cfg->d_c, dr = cfg->d_rope, dm = cfg->d_model;
  const int row = dc + dr, G = gate_width(cfg);
  const int dq = dh + dr;
  const CacheView cv = cache_view(cfg, cache);
  int* status = static_cast<int*>(workspace);
  const bool f32 = cfg->dtype == GMLA_FP32;
  void* cq = static_cast<uint8_t*>(workspace) + 256;   // c^Q [T, d_cq] when the query is compressed

  // GEMM over x: [W_c | W_kr | W_q | W_qr | W_g], or [W_c | W_kr | W_dq | W_g] with a
  // compressed query ("精读笔记 03" §5.1: c^Q = W^DQ h), whose second GEMM reads c^Q:
  // [W_uq | W_qr] (q = W^UQ c^Q; §5.2: q^R = RoPE(W^QR c^Q)).
  const EpiSeg e_q = plain_seg(q_out, static_cast<int64_t>(H) * dq, dh, dq, 0, f32, nullptr, false, false);
  const EpiSeg e_qr = plain_seg(q_out, static_cast<int64_t>(H) * dq, dr, dq, dh, f32, nullptr, true, false);
  ProjSeg segs[kMaxSeg];
  int ns = 0;
  EpiSeg e_c = plain_seg(cache->data, row, 1 << 30, 0, 0, f32, nullptr, false, true);
  EpiSeg e_kr = plain_seg(cache->data, row, dr, 0, dc, f32, nullptr, true, true);
  if (cfg->cache_dtype == GMLA_CACHE_FP8_E4M3) {   // the cache stores E4M3 codes of value / cache_scale
    e_c.out_fp8 = e_kr.out_fp8 = 1;
    e_c.out_scale = e_kr.out_scale = 1.f / cfg->cache_scale;
  }
  segs[ns++] = {w->W_c, dc, e_c};
  if (dr) segs[ns++] = {w->W_kr, dr, e_kr};
  if (compressed) {
    segs[ns++] = {w->W_dq, cfg->d_cq, plain_seg(cq, cfg->d_cq, 1 << 30, 0, 0, f32, nullptr, false, false)};
  } else {
    segs[ns++] = {w->W_q, H * dh, e_q};
    if (dr) segs[ns++] = {w->W_qr, H * dr, e_qr};
  }
  segs[ns++] = {w->W_g, G,
                plain_seg(gate_logits, G, 1 << 30, 0, 0, true, cfg->gate_bias ? w->b_g : nullptr, false, false)};
  GMLA_TRY(project_gemm(cfg, x, T, dm, segs, ns, positions, seq_ids, cv, status, st, "gemm_project"));
  if (!compressed) return GMLA_OK;
  ProjSeg qsegs[2];
  int nq = 0;
  qsegs[nq++] = {w->W_uq, H * dh, e_q};
  if (dr) qsegs[nq++] = {w->W_qr, H * dr, e_qr};
  return project_gemm(cfg, cq, T, cfg->d_cq, qsegs, nq, positions, seq_ids, cv, status, st, "gemm_query_up");
}

// ---------------------------------------------------------------------------
// gmla_decode, and the context-parallel share of it (positions [seq_starts[b],
// seq_lens[b]) written as partials instead of o_gated) for gmla_decode_partial.
static gmla_status decode_impl(const gmla_config* cfg, const gmla_weights* w, const void* q,
                               const float* gate_logits, const gmla_cache* cache, const int32_t* seq_starts,
                               const int32_t* seq_lens, int32_t B, void* o_gated, float* partial_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  GMLA_TRY(check_cfg(cfg));
  if (!w) return fail(GMLA_ERR_INVALID_ARG, "weights is NULL");
  if (B < 0) return fail(GMLA_ERR_INVALID_ARG, "B < 0");
  GMLA_TRY(check_cache(cfg, cache));
  const size_t need = gmla_decode_workspace_size(cfg, B);
  if (!workspace || workspace_bytes < need)
    return fail(GMLA_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need, workspace_bytes);
  GMLA_TRY(check_ptr(workspace, "workspace"));
  if (B == 0) return GMLA_OK;
  if (B > cache->batch) return fail(GMLA_ERR_INVALID_ARG, "B (%d) exceeds cache.batch (%d)", B, cache->batch);
  GMLA_TRY(check_ptr(q, "q"));
  GMLA_TRY(check_ptr(seq_lens, "seq_lens"));
  GMLA_TRY(check_ptr(seq_starts, "seq_starts", false));
  if (partial_out) {
    GMLA_TRY(check_ptr(partial_out, "partial"));
  } else {
    GMLA_TRY(check_ptr(o_gated, "o_gated"));
  }
  GMLA_TRY(check_ptr(gate_logits, "gate_logits", false));
  GMLA_TRY(check_ptr(w->W_k, "W_k"));
  if (!partial_out) GMLA_TRY(check_ptr(w->W_v, "W_v"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const CacheView cv = cache_view(cfg, cache);
  int* status = static_cast<int*>(workspace);

  if (cfg->dtype == GMLA_FP32 && (partial_out || seq_starts))
    return fail(GMLA_ERR_UNSUPPORTED, "context-parallel decode covers the bf16 path");
  if (cfg->dtype == GMLA_FP32) {
    AttnF32Args a{};
    a.q = static_cast<const float*>(q);
    a.cache = static_cast<const float*>(cache->data);
    a.cv = cv;
    a.W_k = static_cast<const float*>(w->W_k);
    a.W_v = static_cast<const float*>(w->W_v);
    a.gate_logits = gate_logits;
    a.o = static_cast<float*>(o_gated);
    a.cu_seqlens = nullptr;
    a.seq_lens = seq_lens;
    a.B = B;
    a.T = B;
    a.H = cfg->n_heads;
    a.d_h = cfg->d_h;
    a.d_c = cfg->d_c;
    a.d_rope = cfg->d_rope;
    a.gate_mode = cfg->gate_mode;
    a.gate_topk = cfg->gate_topk;
    a.scale = cfg->softmax_scale;
    a.status = status;
    cudaError_t e = launch_attn_f32(a, st);
    return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "decode (fp32)");
  }

  if (cfg->d_c != 512 || (cfg->d_rope != 0 && cfg->d_rope != 64))
    return fail(GMLA_ERR_UNSUPPORTED, "bf16 decode covers d_c = 512 with d_rope in {0, 64}");
  if (cfg->d_h != 128 && cfg->d_h != 256) return fail(GMLA_ERR_UNSUPPORTED, "bf16 decode covers d_h in {128, 256}");
  const bool fp8 = cfg->cache_dtype == GMLA_CACHE_FP8_E4M3;
  if (fp8 && (cfg->d_rope != 0 || cfg->d_c != 512))
    return fail(GMLA_ERR_UNSUPPORTED, "an FP8 cache covers NoPE decode with d_c = 512");
  const DecodeLayout L = decode_layout(B, cfg->n_heads, decode_eff_heads(cfg), cfg->d_h, cfg->d_c, cfg->d_rope,
                                       num_sms(), fp8);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeArgs a{};
  const int row = cfg->d_c + cfg->d_rope;
  const int tile_rows = 128;   // tokens per attention tile
  if (fp8) {
    // codes: [rows, row] bytes, boxes of 128 tokens x 128 latent dims
    const bool okm = !cache->paged
                         ? make_tmap_2d_u8(&a.cache_map, cache->data, row,
                                           static_cast<uint64_t>(cache->batch) * cache->capacity, row, 128, tile_rows)
                         : make_tmap_3d_u8(&a.cache_map, cache->data, row, cache->page_size, cache->num_pages, row,
                                           static_cast<uint64_t>(row) * cache->page_size, 128,
                                           cache->page_size < tile_rows ? cache->page_size : tile_rows, 1);
    if (!okm) return fail(GMLA_ERR_CUDA, "tensor map for the FP8 cache failed");
  } else if (!cache->paged) {
    if (!make_tmap_2d(&a.cache_map, cache->data, row, static_cast<uint64_t>(cache->batch) * cache->capacity,
                      static_cast<uint64_t>(row) * 2, 64, tile_rows, true))
      return fail(GMLA_ERR_CUDA, "tensor map for the cache failed");
  } else {
    const int ps = cache->page_size;
    if (!make_tmap_3d(&a.cache_map, cache->data, row, ps, cache->num_pages, static_cast<uint64_t>(row) * 2,
                      static_cast<uint64_t>(row) * 2 * ps, 64, ps < tile_rows ? ps : tile_rows, 1, true))
      return fail(GMLA_ERR_CUDA, "tensor map for the paged cache failed");
  }
  if (fp8 ? !make_tmap_2d_u8(&a.qa_map, ws + L.off_qa, cfg->d_c, static_cast<uint64_t>(B) * L.n_hg * 2 * L.HG,
                             cfg->d_c, 128, 2 * L.HG)
          : !make_tmap_2d(&a.qa_map, ws + L.off_qa, row, static_cast<uint64_t>(B) * cfg->n_heads,
                          static_cast<uint64_t>(row) * 2, 64, L.HG, true))
    return fail(GMLA_ERR_CUDA, "tensor map for the absorbed queries failed");
  if (!fp8) {
    // the tensor-core absorb: W_k as [H*d_h, d_c] in boxes of [d_h x 64], the
    // queries as [B, H*(d_h + d_R)] in boxes of [absorb_bn x 64]
    const int dq = cfg->d_h + cfg->d_rope;
    a.absorb_bn = absorb_tile_n(B);
    if (!make_tmap_2d(&a.wk_map, w->W_k, cfg->d_c, static_cast<uint64_t>(cfg->n_heads) * cfg->d_h,
                      static_cast<uint64_t>(cfg->d_c) * 2, 64, cfg->d_h, true) ||
        !make_tmap_2d(&a.q_map, q, static_cast<uint64_t>(cfg->n_heads) * dq, B,
                      static_cast<uint64_t>(cfg->n_heads) * dq * 2, 64, a.absorb_bn, true))
      return fail(GMLA_ERR_CUDA, "tensor maps for the query absorption failed");
  }
  a.cache = cv;
  a.seq_lens = seq_lens;
  a.q = q;
  a.W_k = w->W_k;
  a.W_v = w->W_v;
  a.gate_logits = gate_logits;
  a.o = o_gated;
  a.qa = ws + L.off_qa;
  a.o_part = reinterpret_cast<float*>(ws + L.off_opart);
  a.ml_part = reinterpret_cast<float*>(ws + L.off_ml);
  a.seg_info = reinterpret_cast<int4*>(ws + L.off_seg);
  a.seq_first_seg = reinterpret_cast<int32_t*>(ws + L.off_seqfirst);
  a.cta_first_seg = reinterpret_cast<int32_t*>(ws + L.off_ctafirst);
  a.status = status;
  a.B = B;
  a.H = cfg->n_heads;
  a.d_h = cfg->d_h;
  a.d_c = cfg->d_c;
  a.d_rope = cfg->d_rope;
  a.gate_mode = cfg->gate_mode;
  a.HG = L.HG;
  a.n_hg = L.n_hg;
  a.G = L.G;
  a.max_seg = L.max_seg;
  a.q_scale = cfg->softmax_scale * 1.4426950408889634f;
  a.test_stall = g_test_stall.exchange(0);
  a.gate_hard = (gate_is_hard(cfg->gate_mode) && gate_logits) ? 1 : 0;
  a.gate_topk = cfg->gate_topk;
  a.gvals = reinterpret_cast<float*>(ws + L.off_gvals);
  a.head_of_slot = reinterpret_cast<int32_t*>(ws + L.off_hslot);
  a.n_act = reinterpret_cast<int32_t*>(ws + L.off_nact);
  a.seq_starts = seq_starts;
  a.partial_out = partial_out;
  a.fp8 = fp8 ? 1 : 0;
  a.cache_scale = cfg->cache_scale;
  a.qmul = reinterpret_cast<float*>(ws + L.off_qmul);
  a.olat = ws + L.off_olat;
  const SwapPlan& sp = L.gemm_plan;
  a.gemm_counters = nullptr;
  a.n_gemm_tiles = 0;

  // o = sigmoid(g) ⊙ W_v^(h) O_lat^(h): a swap-orientation GEMM over heads
  const int HD = cfg->n_heads * cfg->d_h;
  const int G = gate_width(cfg);
  GemmArgs g{};
  if (!make_tmap_2d(&g.act, a.olat, cfg->d_c, static_cast<uint64_t>(cfg->n_heads) * B,
                    static_cast<uint64_t>(cfg->d_c) * 2, 64, sp.bn, true) ||
      !make_tmap_2d(&g.wt[0], w->W_v, cfg->d_c, HD, static_cast<uint64_t>(cfg->d_c) * 2, 64, 128, true))
    return fail(GMLA_ERR_CUDA, "tensor maps for the W_v product failed");
  g.epi[0] = plain_seg(o_gated, HD, 1 << 30, 0, 0, false, nullptr, false, false);
  // hard / quantised gates: the values the absorb kernel computed, else sigmoid of the logits
  g.epi[0].gate = a.gate_hard ? a.gvals : gate_logits;
  g.epi[0].gate_value = a.gate_hard;
  g.epi[0].gate_stride = G;
  g.epi[0].gate_div = cfg->gate_mode == GMLA_GATE_CHANNEL ? 1 : cfg->d_h;
  g.seg_rows[0] = HD;
  g.seg_tile_begin[0] = 0;
  g.seg_tile_begin[1] = HD / 128;
  g.n_seg = 1;
  g.T = B;
  g.K = cfg->d_c;
  g.row_mode = 2;
  g.rows_per_group = cfg->d_h;
  g.act_group_stride = B;
  g.splits = sp.splits;
  g.kb_per_split = sp.kb_per_split;
  g.status = status;

  cudaError_t e = launch_decode_bf16(a, st);
  if (e == cudaSuccess && !partial_out) e = launch_gemm_bf16(g, true, sp.bn, sp.ttiles, st, "gemm_wv_gate");
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "decode");
}

gmla_status gmla_decode(const gmla_config* cfg, const gmla_weights* w, const void* q, const float* gate_logits,
                        const gmla_cache* cache, const int32_t* seq_lens, int32_t B, void* o_gated,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(cfg, w, q, gate_logits, cache, nullptr, seq_lens, B, o_gated, nullptr, workspace,
                     workspace_bytes, stream);
}

gmla_status gmla_decode_partial(const gmla_config* cfg, const gmla_weights* w, const void* q,
                                const float* gate_logits, const gmla_cache* cache, const int32_t* seq_starts,
                                const int32_t* seq_ends, int32_t B, float* partial, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!partial && B > 0) return fail(GMLA_ERR_INVALID_ARG, "partial is NULL");
  return decode_impl(cfg, w, q, gate_logits, cache, seq_starts, seq_ends, B, nullptr, partial, workspace,
                     workspace_bytes, stream);
}

size_t gmla_decode_merge_workspace_size(const gmla_config* cfg, int32_t B) {
  if (!cfg_valid(cfg) || B < 0) return 256;
  const size_t olat = align256(static_cast<size_t>(cfg->n_heads) * B * cfg->d_c * 2);
  const size_t gv = align256(static_cast<size_t>(B) * cfg->n_heads * 4);
  return 256 + olat + gv;
}

gmla_status gmla_decode_merge(const gmla_config* cfg, const gmla_weights* w, const float* partials, int32_t R,
                              const float* gate_logits, int32_t B, void* o_gated, void* workspace,
                              size_t workspace_bytes, void* stream) {
  GMLA_TRY(check_cfg(cfg));
  if (!w) return fail(GMLA_ERR_INVALID_ARG, "weights is NULL");
  if (B < 0 || R < 1) return fail(GMLA_ERR_INVALID_ARG, "B < 0 or R < 1");
  const size_t need = gmla_decode_merge_workspace_size(cfg, B);
  if (!workspace || workspace_bytes < need)
    return fail(GMLA_ERR_WORKSPACE, "decode_merge needs %zu workspace bytes, got %zu", need, workspace_bytes);
  GMLA_TRY(check_ptr(workspace, "workspace"));
  if (B == 0) return GMLA_OK;
  if (cfg->dtype != GMLA_BF16 || cfg->d_c != 512 || cfg->d_h % 128)
    return fail(GMLA_ERR_UNSUPPORTED, "context-parallel merge covers bf16 with d_c = 512 and d_h %% 128 == 0");
  GMLA_TRY(check_ptr(partials, "partials"));
  GMLA_TRY(check_ptr(o_gated, "o_gated"));
  GMLA_TRY(check_ptr(gate_logits, "gate_logits", false));
  GMLA_TRY(check_ptr(w->W_v, "W_v"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int H = cfg->n_heads, HD = H * cfg->d_h, G = gate_width(cfg);
  void* olat = ws + 256;
  float* gvals = reinterpret_cast<float*>(ws + 256 + align256(static_cast<size_t>(H) * B * cfg->d_c * 2));
  MergeRanksArgs m{};
  m.partials = partials;
  m.R = R;
  m.B = B;
  m.H = H;
  m.olat = olat;
  m.gate_logits = gate_logits;
  m.gate_mode = cfg->gate_mode;
  m.gate_topk = cfg->gate_topk;
  m.gate_hard = (gate_is_hard(cfg->gate_mode) && gate_logits) ? 1 : 0;
  m.gvals = gvals;
  cudaError_t e = launch_decode_merge_ranks(m, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode_merge");
  // o = gate ⊙ W_v^(h) O_lat^(h), the same tensor-core GEMM as gmla_decode's
  const SwapPlan sp = gemm_swap_plan(HD / 128, B, cfg->d_c, num_sms());
  GemmArgs g{};
  if (!make_tmap_2d(&g.act, olat, cfg->d_c, static_cast<uint64_t>(H) * B, static_cast<uint64_t>(cfg->d_c) * 2, 64,
                    sp.bn, true) ||
      !make_tmap_2d(&g.wt[0], w->W_v, cfg->d_c, HD, static_cast<uint64_t>(cfg->d_c) * 2, 64, 128, true))
    return fail(GMLA_ERR_CUDA, "tensor maps for the W_v product failed");
  g.epi[0] = plain_seg(o_gated, HD, 1 << 30, 0, 0, false, nullptr, false, false);
  g.epi[0].gate = m.gate_hard ? gvals : gate_logits;
  g.epi[0].gate_value = m.gate_hard;
  g.epi[0].gate_stride = G;
  g.epi[0].gate_div = cfg->gate_mode == GMLA_GATE_CHANNEL ? 1 : cfg->d_h;
  g.seg_rows[0] = HD;
  g.seg_tile_begin[0] = 0;
  g.seg_tile_begin[1] = HD / 128;
  g.n_seg = 1;
  g.T = B;
  g.K = cfg->d_c;
  g.row_mode = 2;
  g.rows_per_group = cfg->d_h;
  g.act_group_stride = B;
  g.splits = sp.splits;
  g.kb_per_split = sp.kb_per_split;
  g.status = static_cast<int*>(workspace);
  e = launch_gemm_bf16(g, true, sp.bn, sp.ttiles, st, "gemm_wv_gate");
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "decode_merge: W_v");
}

// ---------------------------------------------------------------------------
gmla_status gmla_prefill(const gmla_config* cfg, const gmla_weights* w, const void* q, const float* gate_logits,
                         const gmla_cache* cache, const int32_t* cu_seqlens, int32_t B, int32_t T,
                         int32_t max_seqlen, void* o_gated, void* workspace, size_t workspace_bytes,
                         void* stream) {
  GMLA_TRY(check_cfg(cfg));
  if (!w) return fail(GMLA_ERR_INVALID_ARG, "weights is NULL");
  if (B < 0 || T < 0 || max_seqlen < 0) return fail(GMLA_ERR_INVALID_ARG, "negative size");
  GMLA_TRY(check_cache(cfg, cache));
  const size_t need = gmla_prefill_workspace_size(cfg, T, B);
  if (!workspace || workspace_bytes < need)
    return fail(GMLA_ERR_WORKSPACE, "prefill needs %zu workspace bytes, got %zu", need, workspace_bytes);
  GMLA_TRY(check_ptr(workspace, "workspace"));
  if (B == 0 || T == 0) return GMLA_OK;
  if (B > cache->batch) return fail(GMLA_ERR_INVALID_ARG, "B (%d) exceeds cache.batch (%d)", B, cache->batch);
  if (cache->paged) return fail(GMLA_ERR_UNSUPPORTED, "prefill reads a contiguous cache");
  if (cfg->cache_dtype == GMLA_CACHE_FP8_E4M3)
    return fail(GMLA_ERR_UNSUPPORTED, "prefill reads a bf16 or fp32 cache (an FP8 cache is read by decode)");
  if (max_seqlen > cache->capacity) return fail(GMLA_ERR_INVALID_ARG, "max_seqlen exceeds cache.capacity");
  GMLA_TRY(check_ptr(q, "q"));
  GMLA_TRY(check_ptr(cu_seqlens, "cu_seqlens"));
  GMLA_TRY(check_ptr(o_gated, "o_gated"));
  GMLA_TRY(check_ptr(gate_logits, "gate_logits", false));
  GMLA_TRY(check_ptr(w->W_k, "W_k"));
  GMLA_TRY(check_ptr(w->W_v, "W_v"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  const CacheView cv = cache_view(cfg, cache);

  if (cfg->dtype == GMLA_FP32) {
    AttnF32Args a{};
    a.q = static_cast<const float*>(q);
    a.cache = static_cast<const float*>(cache->data);
    a.cv = cv;
    a.W_k = static_cast<const float*>(w->W_k);
    a.W_v = static_cast<const float*>(w->W_v);
    a.gate_logits = gate_logits;
    a.o = static_cast<float*>(o_gated);
    a.cu_seqlens = cu_seqlens;
    a.seq_lens = nullptr;
    a.B = B;
    a.T = T;
    a.H = cfg->n_heads;
    a.d_h = cfg->d_h;
    a.d_c = cfg->d_c;
    a.d_rope = cfg->d_rope;
    a.gate_mode = cfg->gate_mode;
    a.gate_topk = cfg->gate_topk;
    a.max_len = max_seqlen;
    a.scale = cfg->softmax_scale;
    a.status = status;
    cudaError_t e = launch_attn_f32(a, st);
    return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "prefill (fp32)");
  }

  if (cfg->d_rope != 0 && cfg->d_rope != 64)
    return fail(GMLA_ERR_UNSUPPORTED, "bf16 prefill covers NoPE or decoupled RoPE of 64 dims");
  if (cfg->d_h != 128) return fail(GMLA_ERR_UNSUPPORTED, "bf16 prefill covers d_h = 128");
  if (cfg->d_c % 64) return fail(GMLA_ERR_UNSUPPORTED, "bf16 prefill needs d_c %% 64 == 0");
  const int H = cfg->n_heads, HD = H * cfg->d_h;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t kv_bytes = align256(static_cast<size_t>(T) * HD * 2);
  void* Kbuf = ws + 256;
  void* Vbuf = ws + 256 + kv_bytes;

  // K^(h), V^(h) = C W_k^(h)T, C W_v^(h)T for every prompt token
  GemmArgs g{};
  const int bn = 256;
  const int tps = (max_seqlen + 127) / 128;
  if (!make_tmap_2d(&g.act, cache->data, cfg->d_c, static_cast<uint64_t>(cache->batch) * cache->capacity,
                    static_cast<uint64_t>(cv.row) * 2, 64, 128, true))
    return fail(GMLA_ERR_CUDA, "tensor map for cache latents failed");
  const void* Ws[2] = {w->W_k, w->W_v};
  void* outs[2] = {Kbuf, Vbuf};
  g.seg_tile_begin[0] = 0;
  for (int i = 0; i < 2; ++i) {
    if (!make_tmap_2d(&g.wt[i], Ws[i], cfg->d_c, HD, static_cast<uint64_t>(cfg->d_c) * 2, 64, bn, true))
      return fail(GMLA_ERR_CUDA, "tensor map for W_k/W_v failed");
    g.epi[i] = plain_seg(outs[i], HD, 1 << 30, 0, 0, false, nullptr, false, false);
    g.seg_rows[i] = HD;
    g.seg_tile_begin[i + 1] = g.seg_tile_begin[i] + (HD + bn - 1) / bn;
  }
  g.n_seg = 2;
  g.T = T;
  g.K = cfg->d_c;
  g.row_mode = 1;
  g.tiles_per_seq = tps;
  g.act_seq_stride = cache->capacity;
  g.cu_seqlens = cu_seqlens;
  g.status = status;
  cudaError_t e = launch_gemm_bf16(g, false, bn, B * tps, st, "gemm_kv");
  if (e != cudaSuccess) return cuda_fail(e, "prefill K/V rebuild");

  PrefillArgs p{};
  const int dq = cfg->d_h + cfg->d_rope;
  if (!make_tmap_2d(&p.q_map, q, static_cast<uint64_t>(H) * dq, T, static_cast<uint64_t>(H) * dq * 2, 64, 128, true) ||
      !make_tmap_2d(&p.k_map, Kbuf, HD, T, static_cast<uint64_t>(HD) * 2, 64, 128, true) ||
      !make_tmap_2d(&p.v_map, Vbuf, HD, T, static_cast<uint64_t>(HD) * 2, 64, 128, true))
    return fail(GMLA_ERR_CUDA, "tensor maps for prefill attention failed");
  // decoupled RoPE: k^R is read from the cache rows (its last d_R columns)
  if (cfg->d_rope &&
      !make_tmap_2d(&p.kr_map, cache->data, cv.row, static_cast<uint64_t>(cache->batch) * cache->capacity,
                    static_cast<uint64_t>(cv.row) * 2, 64, 128, true))
    return fail(GMLA_ERR_CUDA, "tensor map for the cached k^R failed");
  p.d_c = cfg->d_c;
  p.d_rope = cfg->d_rope;
  p.cache_capacity = cache->capacity;
  p.gate_logits = gate_logits;
  p.o = o_gated;
  p.cu_seqlens = cu_seqlens;
  p.status = status;
  p.B = B;
  p.T = T;
  p.H = H;
  p.d_h = cfg->d_h;
  p.gate_mode = cfg->gate_mode;
  p.gate_topk = cfg->gate_topk;
  p.q_tiles_per_seq = tps;
  p.scale_log2 = cfg->softmax_scale * 1.4426950408889634f;
  e = launch_prefill_attn_bf16(p, st);
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "prefill attention");
}

// ---------------------------------------------------------------------------
gmla_status gmla_gate_out(const gmla_config* cfg, const gmla_weights* w, const void* o, int32_t T,
                          const float* gate_logits, void* y, void* workspace, size_t workspace_bytes,
                          void* stream) {
  GMLA_TRY(check_cfg(cfg));
  if (!w) return fail(GMLA_ERR_INVALID_ARG, "weights is NULL");
  if (T < 0) return fail(GMLA_ERR_INVALID_ARG, "T < 0");
  const size_t need = gmla_gate_out_workspace_size(cfg, T);
  if (!workspace || workspace_bytes < need)
    return fail(GMLA_ERR_WORKSPACE, "gate_out needs %zu workspace bytes, got %zu", need, workspace_bytes);
  GMLA_TRY(check_ptr(workspace, "workspace"));
  if (T == 0) return GMLA_OK;
  GMLA_TRY(check_ptr(o, "o"));
  GMLA_TRY(check_ptr(y, "y"));
  GMLA_TRY(check_ptr(w->W_o, "W_o"));
  GMLA_TRY(check_ptr(gate_logits, "gate_logits", false));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int HD = cfg->n_heads * cfg->d_h, dm = cfg->d_model;
  const bool f32 = cfg->dtype == GMLA_FP32;
  int* status = static_cast<int*>(workspace);
  const void* src = o;
  if (gate_logits) {
    void* tmp = static_cast<uint8_t*>(workspace) + 256;
    cudaError_t e = launch_gate_apply(o, gate_logits, tmp, T, cfg->n_heads, cfg->d_h, cfg->gate_mode, cfg->gate_topk,
                                      f32, st);
    if (e != cudaSuccess) return cuda_fail(e, "gate_out: gate");
    src = tmp;
  }
  const EpiSeg ep = plain_seg(y, dm, 1 << 30, 0, 0, f32, nullptr, false, false);
  if (f32) {
    F32Args a{};
    a.x = static_cast<const float*>(src);
    a.T = T;
    a.K = HD;
    a.W[0] = static_cast<const float*>(w->W_o);
    a.epi[0] = ep;
    a.seg_rows[0] = dm;
    a.n_seg = 1;
    a.status = status;
    cudaError_t e = launch_gemm_f32(a, st);
    return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "gate_out (fp32)");
  }
  if (HD % 8) return fail(GMLA_ERR_UNSUPPORTED, "bf16 path needs H*d_h %% 8 == 0");
  GemmArgs a{};
  const bool swap = T <= 256;
  const SwapPlan sp = gemm_swap_plan((dm + 127) / 128, T, HD, num_sms());
  const int bn = swap ? sp.bn : 256;
  const int wtile = gemm_weight_tile(swap, bn);
  if (!make_tmap_2d(&a.act, src, HD, T, static_cast<uint64_t>(HD) * 2, 64, swap ? bn : 128, true) ||
      !make_tmap_2d(&a.wt[0], w->W_o, HD, dm, static_cast<uint64_t>(HD) * 2, 64, wtile, true))
    return fail(GMLA_ERR_CUDA, "tensor maps for gate_out failed");
  a.epi[0] = ep;
  a.seg_rows[0] = dm;
  a.seg_tile_begin[0] = 0;
  a.seg_tile_begin[1] = (dm + wtile - 1) / wtile;
  a.n_seg = 1;
  a.T = T;
  a.K = HD;
  a.row_mode = 0;
  a.status = status;
  const int ttiles = swap ? sp.ttiles : (T + 127) / 128;
  if (swap) {
    a.splits = sp.splits;
    a.kb_per_split = sp.kb_per_split;
  }
  cudaError_t e = launch_gemm_bf16(a, swap, bn, ttiles, st, "gemm_out");
  return e == cudaSuccess ? GMLA_OK : cuda_fail(e, "gate_out");
}

}  // extern "C"
