// common.cuh — types shared by the kernels and the C-ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gmla {

// Latent cache as the kernels see it (rows of `row` elements).
struct CacheView {
  void* data;
  const int32_t* block_table;
  int32_t paged;
  int32_t batch;
  int32_t capacity;
  int32_t page_size;
  int32_t num_pages;
  int32_t max_pages_per_seq;
  int32_t row;          // d_c + d_R
};

// Global row index of token `pos` of sequence `b`, or -1 when out of range.
static __device__ __noinline__ int64_t cache_row(const CacheView& c, int b, int pos) {
  if (b < 0 || pos < 0) return -1;
  if (!c.paged) {
    if (b >= c.batch || pos >= c.capacity) return -1;
    return static_cast<int64_t>(b) * c.capacity + pos;
  }
  const int pi = pos / c.page_size;
  if (b >= c.batch || pi >= c.max_pages_per_seq) return -1;
  const int page = c.block_table[static_cast<int64_t>(b) * c.max_pages_per_seq + pi];
  if (page < 0 || page >= c.num_pages) return -1;
  return static_cast<int64_t>(page) * c.page_size + (pos % c.page_size);
}

// Gate modes (gmla_gate_mode): per channel, or per head as a sigmoid, hard
// top-k, binary or ternary value.
enum : int { kGateChannel = 0, kGateHead = 1, kGateTopk = 2, kGateBinary = 3, kGateTernary = 4 };

__host__ __device__ inline bool gate_is_hard(int mode) { return mode >= kGateTopk; }

// Gate value of head h of one token from its H per-head logits z
// ("Gated Multi-head Latent Attention", "Gating Mechanism" and "Variants /
// Extensions"): sigmoid(z_h); top-k: 1 for the k largest logits, equal logits
// to the lower head; binary: 1 where sigmoid(z) >= 1/2, i.e. z >= 0; ternary:
// sigmoid(z) rounded to the nearest of 0, 1/2, 1 (halves up), i.e. cut at
// z = -ln 3 and z = ln 3.
__device__ __forceinline__ float head_gate(const float* z, int H, int h, int mode, int k) {
  const float zh = z[h];
  if (mode == kGateTopk) {
    int rank = 0;
    for (int j = 0; j < H; ++j) {
      const float zj = z[j];
      rank += (zj > zh) || (zj == zh && j < h);
    }
    return rank < k ? 1.f : 0.f;
  }
  if (mode == kGateBinary) return zh >= 0.f ? 1.f : 0.f;
  if (mode == kGateTernary) {
    const float ln3 = 1.0986122886681098f;
    return zh < -ln3 ? 0.f : (zh < ln3 ? 0.5f : 1.f);
  }
  return 1.f / (1.f + expf(-zh));
}

// Slot of head h when a token's heads are reordered so that those whose gate
// is not 0 come first (decode computes only those). Top-k: the rank of the
// logit; otherwise active heads by index, then the others by index. *n_act
// gets the number of active heads.
__device__ __forceinline__ int head_slot(const float* z, int H, int h, int mode, int k, int* n_act) {
  if (mode == kGateTopk) {
    int rank = 0;
    for (int j = 0; j < H; ++j) {
      const float zj = z[j], zh = z[h];
      rank += (zj > zh) || (zj == zh && j < h);
    }
    *n_act = k;
    return rank;
  }
  int act = 0, before_act = 0, before_off = 0;
  for (int j = 0; j < H; ++j) {
    const bool on = head_gate(z, H, j, mode, k) != 0.f;
    act += on;
    if (j < h) {
      before_act += on;
      before_off += !on;
    }
  }
  *n_act = act;
  return head_gate(z, H, h, mode, k) != 0.f ? before_act : act + before_off;
}

// How a GEMM epilogue writes one weight segment's outputs.
// Element (token t, feature f) goes to
//   out + row(t) * row_stride + (f / block) * block_stride + (f % block) + col_offset
// where row(t) = t, or the cache row of (seq_ids[t], positions[t]) when
// `cache_scatter` is set. With `rope`, features (2i, 2i+1) of each block are
// rotated by positions[t] * base^(-2i/block) first.
struct EpiSeg {
  void* out;
  const float* bias;     // fp32 [rows] or null
  int64_t row_stride;
  int32_t block;
  int32_t block_stride;
  int32_t col_offset;
  int32_t out_f32;       // 1: fp32 output, 0: bf16 output
  int32_t out_fp8;       // 1: FP8 E4M3 output of v * out_scale (an FP8 latent cache)
  float out_scale;
  int32_t rope;
  int32_t cache_scatter;
  // optional gate: v *= sigmoid(gate[t * gate_stride + f / gate_div]), or with
  // gate_value set v *= gate[...] (gate values computed beforehand)
  const float* gate;
  int32_t gate_stride;
  int32_t gate_div;
  int32_t gate_value;
};

constexpr int kMaxSeg = 5;

struct GemmArgs {
  CUtensorMap act;               // [T rows, K] bf16, box {64, token tile}
  CUtensorMap wt[kMaxSeg];       // per segment [rows, K] bf16, box {64, weight tile}
  EpiSeg epi[kMaxSeg];
  int32_t seg_rows[kMaxSeg];
  int32_t seg_tile_begin[kMaxSeg + 1];
  int32_t n_seg;
  int32_t T;
  int32_t K;
  // row_mode 2: per-group activations (swap orientation): the weight rows of
  //   group g = wrow / rows_per_group read activation rows g*act_group_stride + token.
  int32_t rows_per_group;
  int32_t act_group_stride;
  // row_mode 0: token tile y covers packed tokens [y*tile, ...).
  // row_mode 1: prefill sequence tiles: y -> (sequence y / tiles_per_seq,
  //   offset (y % tiles_per_seq) * tile); activation rows start at
  //   sequence * act_seq_stride, packed tokens at cu_seqlens[sequence].
  int32_t row_mode;
  // split-K (swap orientation only): blockIdx.z is the split; each split
  // accumulates kb_per_split 64-wide K blocks; the splits of a tile run as one
  // cluster and rank 0 sums their partials through distributed shared memory.
  int32_t splits;
  int32_t kb_per_split;
  int32_t tiles_per_seq;
  int32_t act_seq_stride;
  const int32_t* cu_seqlens;
  const int32_t* positions;
  const int32_t* seq_ids;
  CacheView cache;
  double log2_rope_base;
  int* status;
};

// RoPE of one element given its pair partner: pair (x0, x1) at feature
// (2i, 2i+1) becomes (x0 cos - x1 sin, x0 sin + x1 cos), angle pos * base^(-2i/d).
// The angle is formed and reduced in double so long positions keep their accuracy.
static __device__ __noinline__ float rope_rotate(float v, float partner, bool odd, int pos, int i_pair, int d,
                                          double log2_base) {
  const double inv = exp2(-(2.0 * i_pair / d) * log2_base);
  double ang = static_cast<double>(pos) * inv;
  ang -= 6.283185307179586476925 * rint(ang * 0.159154943091895335768883763);
  float s, c;
  sincosf(static_cast<float>(ang), &s, &c);
  return odd ? (partner * s + v * c) : (v * c - partner * s);
}

// One output element of an epilogue in the segment's format: fp32, bf16, or an
// FP8 E4M3 code of v * out_scale (round to nearest even, saturating).
__device__ __forceinline__ void store_out(const EpiSeg& e, int64_t off, float v) {
  if (e.out_f32)
    static_cast<float*>(e.out)[off] = v;
  else if (e.out_fp8)
    static_cast<uint8_t*>(e.out)[off] =
        static_cast<uint8_t>(__nv_cvt_float_to_fp8(v * e.out_scale, __NV_SATFINITE, __NV_E4M3));
  else
    static_cast<__nv_bfloat16*>(e.out)[off] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ void epi_store(const EpiSeg& e, int64_t row, int f, float v, int t = 0) {
  if (e.gate) {
    const float g = e.gate[static_cast<int64_t>(t) * e.gate_stride + f / e.gate_div];
    v *= e.gate_value ? g : __fdividef(1.f, 1.f + __expf(-g));
  }
  const int64_t off = row * e.row_stride + static_cast<int64_t>(f / e.block) * e.block_stride + (f % e.block) +
                      e.col_offset;
  if (e.bias) v += e.bias[f];
  store_out(e, off, v);
}

}  // namespace gmla
