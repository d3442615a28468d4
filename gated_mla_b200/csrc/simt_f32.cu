// simt_f32.cu — the fp32 path on CUDA cores, plus the elementwise gate.
//
// fp32 inputs need fp32 arithmetic end to end (tensor-core tf32 would lose the
// 1e-4 agreement), so this path uses FFMA:
//   * launch_gemm_f32: tiled D = X W^T with the same fused epilogues as the
//     tensor-core GEMM (cache scatter, RoPE, q layout, gate logits + bias).
//   * launch_attn_f32: one block per (query token, head), absorbed form
//     ("精读笔记 03" §5.1, 题4): q_lat = W_k^T q, streaming online softmax over
//     the cached rows in chunks, O_lat = sum p c, o = W_v O_lat / l, then the
//     sigmoid gate ("Gated MLA 计算公式" §二 boxed equation).
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gmla {

// ---------------------------------------------------------------------------
// fp32 GEMM with fused epilogue: block = 64 features x 16 tokens; each thread
// owns a feature pair (2i, 2i+1) of one token so RoPE pairs stay in-thread.
// ---------------------------------------------------------------------------
constexpr int kF32FT = 64;    // features per block
constexpr int kF32TT = 16;    // tokens per block
constexpr int kF32KC = 32;    // K chunk

__global__ void __launch_bounds__(512) gemm_f32_kernel(const F32Args a) {
  int s = 0;
  while (s + 1 < a.n_seg && static_cast<int>(blockIdx.x) >= a.seg_tile_begin[s + 1]) ++s;
  const int f0 = (blockIdx.x - a.seg_tile_begin[s]) * kF32FT;
  const int t0 = blockIdx.y * kF32TT;
  const int rows = a.seg_rows[s];
  const float* W = a.W[s];
  __shared__ float sx[kF32TT][kF32KC + 1];
  __shared__ float sw[kF32FT][kF32KC + 1];
  const int tx = threadIdx.x & 31;   // feature pair
  const int ty = threadIdx.x >> 5;   // token
  float acc0 = 0.f, acc1 = 0.f;
  for (int k0 = 0; k0 < a.K; k0 += kF32KC) {
    for (int i = threadIdx.x; i < kF32TT * kF32KC; i += blockDim.x) {
      const int r = i / kF32KC, c = i % kF32KC;
      const int t = t0 + r, k = k0 + c;
      sx[r][c] = (t < a.T && k < a.K) ? a.x[static_cast<int64_t>(t) * a.K + k] : 0.f;
    }
    for (int i = threadIdx.x; i < kF32FT * kF32KC; i += blockDim.x) {
      const int r = i / kF32KC, c = i % kF32KC;
      const int f = f0 + r, k = k0 + c;
      sw[r][c] = (f < rows && k < a.K) ? W[static_cast<int64_t>(f) * a.K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kF32KC; ++c) {
      const float xv = sx[ty][c];
      acc0 = fmaf(xv, sw[2 * tx][c], acc0);
      acc1 = fmaf(xv, sw[2 * tx + 1][c], acc1);
    }
    __syncthreads();
  }
  const int t = t0 + ty;
  const int f = f0 + 2 * tx;
  if (t >= a.T || f >= rows) return;
  const EpiSeg& e = a.epi[s];
  int pos = 0;
  int64_t row = t;
  if (e.rope || e.cache_scatter) pos = a.positions[t];
  if (e.cache_scatter) {
    row = cache_row(a.cache, a.seq_ids[t], pos);
    if (row < 0) {
      report_status(a.status, kStatusRange);
      return;
    }
  }
  float v0 = acc0, v1 = acc1;
  if (e.rope) {
    const int fi = f % e.block;
    v0 = rope_rotate(acc0, acc1, false, pos, fi >> 1, e.block, a.log2_rope_base);
    v1 = rope_rotate(acc1, acc0, true, pos, fi >> 1, e.block, a.log2_rope_base);
  }
  epi_store(e, row, f, v0);
  if (f + 1 < rows) epi_store(e, row, f + 1, v1);
}

cudaError_t launch_gemm_f32(F32Args a, cudaStream_t st) {
  a.seg_tile_begin[0] = 0;
  for (int i = 0; i < a.n_seg; ++i) a.seg_tile_begin[i + 1] = a.seg_tile_begin[i] + (a.seg_rows[i] + kF32FT - 1) / kF32FT;
  const int nx = a.seg_tile_begin[a.n_seg];
  if (nx == 0 || a.T == 0) return cudaSuccess;
  prof_begin(st, "gemm_f32");
  gemm_f32_kernel<<<dim3(nx, (a.T + kF32TT - 1) / kF32TT), 512, 0, st>>>(a);
  prof_end(st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// fp32 attention, one block per (query, head)
// ---------------------------------------------------------------------------
constexpr int kAttnThreads = 256;
constexpr int kChunk = 256;        // keys per online-softmax step
constexpr int kMaxDc = 1024;

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r += red[i];
  return r;
}

__global__ void __launch_bounds__(kAttnThreads) attn_f32_kernel(const AttnF32Args a) {
  const int qi = blockIdx.x, h = blockIdx.y;
  const int dq = a.d_h + a.d_rope, row = a.d_c + a.d_rope;
  int b, t, nkeys;
  if (a.cu_seqlens) {
    b = 0;
    while (b + 1 < a.B && a.cu_seqlens[b + 1] <= qi) ++b;
    t = qi - a.cu_seqlens[b];
    nkeys = t + 1;
  } else {
    b = qi;
    nkeys = a.seq_lens[b];
    t = nkeys - 1;
  }
  const int limit = a.cv.paged ? a.cv.max_pages_per_seq * a.cv.page_size : a.cv.capacity;
  __shared__ float sq[512];
  __shared__ float sqlat[kMaxDc];
  __shared__ float sp[kChunk];
  __shared__ float red[32];
  const int HD = a.H * a.d_h;
  const int G = a.gate_mode == 0 ? HD : a.H;
  float* out = a.o + static_cast<int64_t>(qi) * HD + h * a.d_h;
  if (nkeys <= 0 || nkeys > limit || b >= a.cv.batch) {
    if (nkeys != 0 && threadIdx.x == 0) report_status(a.status, kStatusRange);
    for (int i = threadIdx.x; i < a.d_h; i += blockDim.x) out[i] = 0.f;
    return;
  }
  // per-head gates are one value per (token, head); a head whose gate is 0 is skipped
  float gh = 1.f;
  if (a.gate_logits && a.gate_mode != 0) {
    gh = head_gate(a.gate_logits + static_cast<int64_t>(qi) * G, a.H, h, a.gate_mode, a.gate_topk);
    if (gh == 0.f) {
      for (int i = threadIdx.x; i < a.d_h; i += blockDim.x) out[i] = 0.f;
      return;
    }
  }
  const float* q = a.q + (static_cast<int64_t>(qi) * a.H + h) * dq;
  for (int i = threadIdx.x; i < dq; i += blockDim.x) sq[i] = q[i];
  __syncthreads();
  // q_lat = W_k^(h)T q
  const float* Wk = a.W_k + static_cast<int64_t>(h) * a.d_h * a.d_c;
  for (int d = threadIdx.x; d < a.d_c; d += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < a.d_h; ++i) acc = fmaf(sq[i], Wk[static_cast<int64_t>(i) * a.d_c + d], acc);
    sqlat[d] = acc;
  }
  __syncthreads();
  const float NEG_INF = -__int_as_float(0x7f800000);
  float m = NEG_INF, l = 0.f;
  float acc[kMaxDc / kAttnThreads];
#pragma unroll
  for (int j = 0; j < kMaxDc / kAttnThreads; ++j) acc[j] = 0.f;
  for (int s0 = 0; s0 < nkeys; s0 += kChunk) {
    const int s = s0 + threadIdx.x;
    float z = NEG_INF;
    if (s < nkeys) {
      const int64_t r = cache_row(a.cv, b, s);
      const float* c = a.cache + r * row;
      float dot = 0.f;
      for (int d = 0; d < a.d_c; ++d) dot = fmaf(sqlat[d], c[d], dot);
      for (int d = 0; d < a.d_rope; ++d) dot = fmaf(sq[a.d_h + d], c[a.d_c + d], dot);
      z = a.scale * dot;
    }
    const float cm = block_reduce_max(z, red);
    const float mn = fmaxf(m, cm);
    const float alpha = (m == NEG_INF) ? 0.f : expf(m - mn);
    const float p = (s < nkeys) ? expf(z - mn) : 0.f;
    sp[threadIdx.x] = p;
    const float ps = block_reduce_sum(p, red);
    l = l * alpha + ps;
    m = mn;
    __syncthreads();
    const int n = min(kChunk, nkeys - s0);
#pragma unroll
    for (int j = 0; j < kMaxDc / kAttnThreads; ++j) {
      const int d = threadIdx.x + j * kAttnThreads;
      if (d >= a.d_c) break;
      float v = acc[j] * alpha;
      for (int k = 0; k < n; ++k) {
        const int64_t r = cache_row(a.cv, b, s0 + k);
        v = fmaf(sp[k], a.cache[r * row + d], v);
      }
      acc[j] = v;
    }
    __syncthreads();
  }
  // O_lat = acc / l  (reuse sqlat)
  const float inv = 1.f / l;
#pragma unroll
  for (int j = 0; j < kMaxDc / kAttnThreads; ++j) {
    const int d = threadIdx.x + j * kAttnThreads;
    if (d < a.d_c) sqlat[d] = acc[j] * inv;
  }
  __syncthreads();
  const float* Wv = a.W_v + static_cast<int64_t>(h) * a.d_h * a.d_c;
  for (int i = threadIdx.x; i < a.d_h; i += blockDim.x) {
    float v = 0.f;
    for (int d = 0; d < a.d_c; ++d) v = fmaf(Wv[static_cast<int64_t>(i) * a.d_c + d], sqlat[d], v);
    if (a.gate_logits) {
      if (a.gate_mode == 0) {
        const float zg = a.gate_logits[static_cast<int64_t>(qi) * G + h * a.d_h + i];
        v *= 1.f / (1.f + expf(-zg));
      } else {
        v *= gh;
      }
    }
    out[i] = v;
  }
}

cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t st) {
  if (a.d_c > kMaxDc || a.d_h + a.d_rope > 512) return cudaErrorInvalidValue;
  if (a.T == 0) return cudaSuccess;
  prof_begin(st, "attn_f32");
  attn_f32_kernel<<<dim3(a.T, a.H), kAttnThreads, 0, st>>>(a);
  prof_end(st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// out = sigmoid(g) ⊙ o  (per channel, or per head broadcast over d_h)
// ---------------------------------------------------------------------------
__global__ void gate_apply_kernel(const void* o, const float* g, void* out, int64_t n, int HD, int H, int d_h,
                                  int is_f32) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float s = 1.f / (1.f + expf(-g[i]));   // per channel: G = HD, same index as o
    if (is_f32) {
      static_cast<float*>(out)[i] = static_cast<const float*>(o)[i] * s;
    } else {
      const float v = __bfloat162float(static_cast<const __nv_bfloat16*>(o)[i]);
      static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v * s);
    }
  }
}

// per-head gates (sigmoid, top-k, binary, ternary): one warp per (token, head),
// the gate value computed once from the token's H logits, lanes over d_h
__global__ void gate_apply_head_kernel(const void* o, const float* g, void* out, int T, int H, int d_h,
                                       int gate_mode, int gate_topk, int is_f32) {
  const int lane = threadIdx.x & 31;
  const int64_t pairs = static_cast<int64_t>(T) * H;
  for (int64_t p = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; p < pairs;
       p += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t t = p / H;
    const int h = static_cast<int>(p % H);
    const float s = head_gate(g + t * H, H, h, gate_mode, gate_topk);
    const int64_t base = p * d_h;
    for (int c = lane; c < d_h; c += 32) {
      if (is_f32) {
        static_cast<float*>(out)[base + c] = static_cast<const float*>(o)[base + c] * s;
      } else {
        const float v = __bfloat162float(static_cast<const __nv_bfloat16*>(o)[base + c]);
        static_cast<__nv_bfloat16*>(out)[base + c] = __float2bfloat16_rn(v * s);
      }
    }
  }
}

cudaError_t launch_gate_apply(const void* o, const float* g, void* out, int T, int H, int d_h, int gate_mode,
                              int gate_topk, int is_f32, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(T) * H * d_h;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  prof_begin(st, "gate_apply");
  if (gate_mode == 0) {
    const int64_t blocks = (n + threads - 1) / threads;
    gate_apply_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), threads, 0, st>>>(o, g, out, n, H * d_h,
                                                                                             H, d_h, is_f32);
  } else {
    const int64_t blocks = (static_cast<int64_t>(T) * H * 32 + threads - 1) / threads;
    gate_apply_head_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), threads, 0, st>>>(
        o, g, out, T, H, d_h, gate_mode, gate_topk, is_f32);
  }
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace gmla
