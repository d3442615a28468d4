// internal.h — declarations shared between the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

struct gmla_config;

namespace gmla {

// Argument check of a configuration shared by the entry points (gmla.cu):
// returns a gmla_status and sets the thread's last error when it fails.
int check_config(const ::gmla_config* c);

// Launches `kernel` with programmatic stream serialization: it may begin
// while the previous kernel of the stream is still running, and calls
// griddep_wait() before it touches data another kernel reads or writes. With
// cluster_z > 1 the blocks form clusters of that size along z.
template <typename Args>
inline cudaError_t launch_pdl(void (*kernel)(Args), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              int cluster_z, const Args& args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = static_cast<unsigned>(cluster_z);
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args);
}

// ----- tcgen05 GEMM (gemm_tc.cu) -----
cudaError_t launch_gemm_bf16(const GemmArgs& a, bool swap, int bn, int token_tiles, cudaStream_t st,
                             const char* name);
int gemm_weight_tile(bool swap, int bn);
int gemm_swap_bn(int T);
// Tiling of the swap orientation (few tokens): token tile width, K splits and
// the workspace they need (ticket counters, then fp32 partial tiles).
struct SwapPlan {
  int bn, ttiles, tiles, splits, kb_per_split;
  size_t ws_bytes;
};
SwapPlan gemm_swap_plan(int wtiles, int T, int K, int num_sms);

// ----- decode (decode_tc.cu) -----
struct DecodeArgs {
  CUtensorMap cache_map;     // contiguous: 2D [B*cap, row]; paged: 3D [pages, page_size, row]
  CUtensorMap qa_map;        // 2D [B*H, row] bf16 absorbed queries
  CUtensorMap wk_map;        // 2D [H*d_h, d_c] bf16 W_k, boxes of [d_h rows x 64 columns] (bf16 cache)
  CUtensorMap q_map;         // 2D [B, H*(d_h + d_R)] bf16 queries, boxes of [absorb_bn rows x 64] (bf16 cache)
  int32_t absorb_bn;         // sequences per absorb CTA (multiple of 16, <= 128)
  CacheView cache;
  const int32_t* seq_lens;   // [B]
  const void* q;             // [B, H, d_h + d_R]
  const void* W_k;           // [H, d_h, d_c]
  const void* W_v;           // [H, d_h, d_c]
  const float* gate_logits;  // [B, G] or null
  void* o;                   // [B, H*d_h]
  void* qa;                  // workspace: [B*H, row] bf16
  float* o_part;             // workspace: [n_hg, max_seg, HG, d_c]
  float* ml_part;            // workspace: [n_hg, max_seg, HG, 2]
  int4* seg_info;            // workspace: [max_seg] {sequence, first tile, end tile, length}
  int32_t* seq_first_seg;    // workspace: [B + 1]
  int32_t* cta_first_seg;    // workspace: [G + 1]
  void* olat;                // workspace: [H, B, d_c] bf16 merged latent outputs
  int32_t* gemm_counters;    // workspace: split-K tickets of the W_v GEMM
  int32_t n_gemm_tiles;
  int* status;
  int32_t B, H, d_h, d_c, d_rope, gate_mode;
  int32_t HG, n_hg, G, max_seg;
  float q_scale;             // softmax_scale * log2(e), folded into the absorbed query
  int32_t test_stall;        // test hook: the first CTA's MMA thread waits on a barrier nothing completes
  // hard / quantised per-head gates: heads whose gate is 0 are skipped. The
  // absorbed queries of sequence b are stored by slot (active heads first);
  // head_of_slot maps a slot back to its head.
  int32_t gate_hard;         // 1: gate_mode is top-k, binary or ternary and gate logits are given
  int32_t gate_topk;
  float* gvals;              // workspace: [B, H] gate values
  int32_t* head_of_slot;     // workspace: [B, H]
  int32_t* n_act;            // workspace: [B] heads whose gate is not 0
  // context-parallel share: attend to positions [seq_starts[b], seq_lens[b]) only
  // (null: from 0), and write per-(sequence, head) partials instead of O_lat
  const int32_t* seq_starts;
  float* partial_out;        // [B, H, d_c + 4]: O_lat / l, then log2-domain m + log2 l
  // FP8 (E4M3) latent cache: codes times cache_scale; the absorbed queries are
  // hi/lo e4m3 rows [B, n_hg, 2, HG, d_c] with one multiplier per (sequence, slot)
  int32_t fp8;
  float cache_scale;
  float* qmul;               // workspace: [B, H] sigma * cache_scale
};

// Cross-rank merge of context-parallel partials into O_lat (bf16 [H, B, d_c]),
// plus the gate values of hard / quantised per-head gates.
struct MergeRanksArgs {
  const float* partials;     // [R, B, H, d_c + 4]
  int32_t R, B, H;
  void* olat;                // [H, B, d_c] bf16
  const float* gate_logits;  // [B, H] (hard gates only) or null
  int32_t gate_mode, gate_topk, gate_hard;
  float* gvals;              // [B, H]
};
cudaError_t launch_decode_merge_ranks(const MergeRanksArgs& a, cudaStream_t st);
constexpr int kPartialPad = 4;   // floats after the d_c values of a partial row

struct DecodeLayout {
  size_t off_qa, off_opart, off_ml, off_seg, off_seqfirst, off_ctafirst, off_olat, off_gemm;
  size_t off_gvals, off_hslot, off_nact, off_qmul, total;
  int HG, n_hg, G, max_seg;
  SwapPlan gemm_plan;        // the W_v GEMM (heads x 128 rows, B tokens, K = d_c)
};
// eff_heads: the most heads a sequence attends with (H, or k with top-k gates),
// which sets the head groups of the attention kernel.
DecodeLayout decode_layout(int B, int H, int eff_heads, int d_h, int d_c, int d_rope, int num_sms, bool fp8 = false);
// sequences per CTA of the tensor-core absorb (N of its MMA)
int absorb_tile_n(int B);
cudaError_t launch_decode_bf16(DecodeArgs& a, cudaStream_t st);

// ----- fp32 CUDA-core path (simt_f32.cu) -----
struct F32Args {
  const float* x;            // [T, K] activations
  int32_t T, K;
  const float* W[kMaxSeg];   // segment weights [rows, K]
  EpiSeg epi[kMaxSeg];
  int32_t seg_rows[kMaxSeg];
  int32_t seg_tile_begin[kMaxSeg + 1];   // filled by launch_gemm_f32
  int32_t n_seg;
  const int32_t* positions;
  const int32_t* seq_ids;
  CacheView cache;
  double log2_rope_base;
  int* status;
};
cudaError_t launch_gemm_f32(F32Args a, cudaStream_t st);

struct AttnF32Args {
  const float* q;            // [T or B, H, d_h + d_R]
  const float* cache;        // cache rows (fp32)
  CacheView cv;
  const float* W_k;
  const float* W_v;
  const float* gate_logits;
  float* o;
  const int32_t* cu_seqlens; // prefill: [B+1]; null for decode
  const int32_t* seq_lens;   // decode: [B]
  int32_t B, T, H, d_h, d_c, d_rope, gate_mode, gate_topk, max_len;
  float scale;
  float* scratch;            // [B*H*(d_c + max_len)] or per-launch scratch
  int* status;
};
cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t st);

// ----- prefill (prefill_tc.cu) -----
struct PrefillArgs {
  CUtensorMap q_map;         // 2D [T, H*(d_h+d_R)] bf16
  CUtensorMap k_map;         // 2D [T, H*d_h] bf16
  CUtensorMap v_map;         // 2D [T, H*d_h] bf16
  CUtensorMap kr_map;        // 2D cache rows [batch*capacity, d_c + d_R] bf16 (decoupled RoPE only)
  int32_t d_c, d_rope, cache_capacity;
  const float* gate_logits;  // [T, G] or null
  void* o;                   // [T, H*d_h]
  const int32_t* cu_seqlens;
  int* status;
  int32_t B, T, H, d_h, gate_mode, gate_topk, q_tiles_per_seq;
  float scale_log2;
};
cudaError_t launch_prefill_attn_bf16(const PrefillArgs& a, cudaStream_t st);

// ----- elementwise helpers (gmla.cu) -----
cudaError_t launch_gate_apply(const void* o, const float* g, void* out, int T, int H, int d_h, int gate_mode,
                              int gate_topk, int is_f32, cudaStream_t st);

// ----- error message of the current host thread (gmla.cu) -----
void set_last_error(const char* msg);

// ----- instrumentation (gmla.cu) -----
// Record a start event (when profiling is on) and count one launch.
void prof_begin(cudaStream_t st, const char* name);
// Record the matching stop event.
void prof_end(cudaStream_t st);

// ----- tensor maps -----
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128);
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box_inner, uint32_t box1,
                  uint32_t box2, bool swizzle128);
// the same over one-byte elements (FP8 codes)
bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                     uint32_t box_inner, uint32_t box_rows);
bool make_tmap_3d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t d1, uint64_t d2,
                     uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box_inner, uint32_t box1,
                     uint32_t box2);

}  // namespace gmla
