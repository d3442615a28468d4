// noalloc.cu — gmla_decode_noalloc: gmla_decode without a caller-provided
// workspace.
//
// Some callers cannot hand the library a device buffer: inference engines and
// plugins whose device memory is owned by their own pool and who forbid
// third-party allocations, and latency-critical loops that cannot pay for
// cudaMalloc's implicit device synchronisation. For them this file keeps the
// decode scratch (status word, absorbed queries, split plan and split-K
// partials) in one file-scope device array instead.
//
// The array is kScratchBytes long and every GPU that loads the library holds
// it until the process exits. Every call shares it and it keeps the previous
// call's contents, so calls whose kernels overlap on the GPU (for example on
// different streams) race on it; serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gmla.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the
// symbol itself is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
gmla_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    gmla::set_last_error("gmla_decode_noalloc: cudaGetDevice failed");
    return GMLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    gmla::set_last_error("gmla_decode_noalloc: device ordinal out of range");
    return GMLA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      gmla::set_last_error("gmla_decode_noalloc: cudaGetSymbolAddress of the static scratch failed");
      return GMLA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GMLA_OK;
}

}  // namespace

extern "C" GMLA_API gmla_status gmla_decode_noalloc(const gmla_config* cfg, const gmla_weights* w, const void* q,
                                                    const float* gate_logits, const gmla_cache* cache,
                                                    const int32_t* seq_lens, int32_t B, void* o_gated,
                                                    void* stream) {
  // the configuration and batch are checked before the scratch size is worked out
  const gmla_status cs = static_cast<gmla_status>(gmla::check_config(cfg));
  if (cs != GMLA_OK) return cs;
  if (B < 0) {
    gmla::set_last_error("gmla_decode_noalloc: B < 0");
    return GMLA_ERR_INVALID_ARG;
  }
  const size_t need = gmla_decode_workspace_size(cfg, B);
  if (need > kScratchBytes) {
    gmla::set_last_error(
        "gmla_decode_noalloc: this batch needs more scratch than the 16 MiB static array holds; "
        "use gmla_decode with a workspace of gmla_decode_workspace_size() bytes");
    return GMLA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  gmla_status s = scratch_address(&scratch);
  if (s != GMLA_OK) return s;
  // the status word must start at zero; everything else is written before it is read
  s = gmla_clear_status(scratch, stream);
  if (s != GMLA_OK) return s;
  return gmla_decode(cfg, w, q, gate_logits, cache, seq_lens, B, o_gated, scratch, kScratchBytes, stream);
}
