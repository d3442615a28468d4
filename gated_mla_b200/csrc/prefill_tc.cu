// prefill_tc.cu — causal attention of whole prompts on tcgen05 tensor cores,
// explicit form ("Gated MLA 计算公式" §一/§二): K^(h), V^(h) were rebuilt from the
// cached latents by the GEMM of gemm_tc.cu; here
//   S = Q K^T (TMEM, fp32)  ->  online softmax over keys s <= t (fp32, registers)
//   O += P V (TMEM, fp32)   ->  o = O / l, gated by sigmoid(g) on the way out.
// One CTA per (128-query tile, head, sequence). Warp 0 loads Q once and K/V
// tiles through a two-stage ring with TMA; one thread of warp 1 issues the
// MMAs; warps 2..5 own one query row per thread for the softmax and epilogue.
// The running max of a row is only raised when a tile's max exceeds it by
// more than 2^8 (the final normalisation uses the same reference, so the
// result is exact); the O row is rescaled in TMEM only then.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gmla {

namespace {
constexpr int kBQ = 128;          // queries per tile
constexpr int kBK = 128;          // keys per tile
constexpr int kD = 128;           // head dim
constexpr int kHalf = kBQ * 128;  // one [128 rows x 64] bf16 box: 16 KB
constexpr int kQBytes = 2 * kHalf;
constexpr int kKVBytes = 2 * kHalf;
constexpr int kStages = 2;
constexpr int kPBytes = 2 * kHalf;
constexpr int kSmem = kQBytes + 2 * kStages * kKVBytes + kPBytes + 1024 + 512;
constexpr uint32_t kTmemCols = 256;

struct PfBars {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, p_full, o_done, drain;
  uint32_t tmem;
  int abort;
};
}  // namespace

__global__ void __launch_bounds__(192, 1) prefill_attn_kernel(const __grid_constant__ PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;                     // [stage][2 boxes]
  uint8_t* sV = sK + kStages * kKVBytes;
  uint8_t* sP = sV + kStages * kKVBytes;
  PfBars* bars = reinterpret_cast<PfBars*>(sP + kPBytes);
  volatile int* abort_flag = &bars->abort;

  const int b = blockIdx.z, h = blockIdx.y;
  const int qt = a.q_tiles_per_seq - 1 - static_cast<int>(blockIdx.x);   // long rows first
  const int beg = a.cu_seqlens[b];
  const int len = a.cu_seqlens[b + 1] - beg;
  const int q0 = qt * kBQ;
  if (q0 >= len) return;
  const int n_kv = qt + 1;                       // causal: key tiles 0..qt
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dq = a.d_h;                          // NoPE: q row is d_h wide per head

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.q_map);
      tma_prefetch_desc(&a.k_map);
      tma_prefetch_desc(&a.v_map);
      const uint64_t pol = l2_evict_last();
      mbar_arrive_expect_tx(&bars->q_full, kQBytes);
      for (int kb = 0; kb < 2; ++kb)
        tma_load_2d(&a.q_map, &bars->q_full, sQ + kb * kHalf, h * dq + kb * 64, beg + q0, pol);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&bars->kv_empty[st], ((j / kStages) & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kKVBytes);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_2d(&a.k_map, &bars->kv_full[st], sK + st * kKVBytes + kb * kHalf, h * kD + kb * 64,
                      beg + j * kBK, pol);
          tma_load_2d(&a.v_map, &bars->kv_full[st], sV + st * kKVBytes + kb * kHalf, h * kD + kb * 64,
                      beg + j * kBK, pol);
        }
        ++issued;
      }
      if (*abort_flag) {
        mbar_drain(&bars->q_full, 0);
        for (int j = max(0, issued - kStages); j < issued; ++j)
          mbar_drain(&bars->kv_full[j % kStages], (j / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);   // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(128, 128, false, true);    // P K-major, V MN-major
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV), pa = smem_u32(sP);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.status);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(&bars->kv_full[st], (j / kStages) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kbase = ka + st * kKVBytes, vbase = va + st * kKVBytes;
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const int kb = k >> 2, kk = k & 3;
          umma_bf16(tS, sdesc_sw128(qa + kb * kHalf + kk * 32, 16, 1024),
                    sdesc_sw128(kbase + kb * kHalf + kk * 32, 16, 1024), idS, k != 0);
        }
        umma_commit(&bars->s_full);
        if (!mbar_wait(&bars->p_full, j & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const int kb = k >> 2, kk = k & 3;
          umma_bf16(tO, sdesc_sw128(pa + kb * kHalf + kk * 32, 16, 1024),
                    sdesc_sw128(vbase + k * 2048, kHalf, 1024), idO, (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&bars->kv_empty[st]);
      }
      if (ok) {
        umma_commit(&bars->o_done);
      } else {
        umma_commit(&bars->drain);
        mbar_drain(&bars->drain, 0);
      }
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // query row in the tile
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int qi = q0 + r;                        // position in the sequence
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m = NEG_INF, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(&bars->s_full, j & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      const bool diag = (j == qt);
      // pass 1: row max of this tile (scaled to log2 units)
      float tmax = NEG_INF;
#pragma unroll
      for (int c = 0; c < kBK; c += 16) {
        uint32_t v[16];
        tmem_ld16(tS + lane_off + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const bool keep = !diag || (c + i <= r);
          if (keep) tmax = fmaxf(tmax, __uint_as_float(v[i]) * a.scale_log2);
        }
      }
      if (j == 0 || tmax > m + 8.f) {
        const float mn = fmaxf(m, tmax);
        const float alpha = (m == NEG_INF) ? 0.f : ex2_approx(m - mn);
        if (j > 0 && alpha != 1.f) {
          // O of the previous tile is complete (S of this tile was issued after it)
#pragma unroll 1
          for (int c = 0; c < kD; c += 16) {
            uint32_t v[16];
            tmem_ld16(tO + lane_off + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st16(tO + lane_off + c, v);
          }
          tmem_st_wait();
        }
        l *= alpha;
        m = mn;
      }
      // pass 2: P = exp2(s*scale - m) -> bf16 K-major [query row][key], two 64-key boxes
#pragma unroll
      for (int c = 0; c < kBK; c += 16) {
        uint32_t v[16];
        tmem_ld16(tS + lane_off + c, v);
        tmem_ld_wait();
        float p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const bool keep = !diag || (c + i <= r);
          p[i] = keep ? ex2_approx(__uint_as_float(v[i]) * a.scale_log2 - m) : 0.f;
          l += p[i];
        }
        uint8_t* box = sP + (c >> 6) * kHalf;
        const int col = c & 63;
#pragma unroll
        for (int i = 0; i < 16; i += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(p[i + 0], p[i + 1]);
          pk.y = pack_bf16x2(p[i + 2], p[i + 3]);
          pk.z = pack_bf16x2(p[i + 4], p[i + 5]);
          pk.w = pack_bf16x2(p[i + 6], p[i + 7]);
          *reinterpret_cast<uint4*>(box + sw128_offset(r, col + i)) = pk;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    if (ok && mbar_wait(&bars->o_done, 0, abort_flag, a.status)) {
      tc_fence_after();
      const bool valid = qi < len;
      const int HD = a.H * kD;
      const int G = a.gate_mode == 0 ? HD : a.H;
      const int64_t tok = beg + qi;
      const float inv = 1.f / l;
      float gh = 1.f;
      if (valid && a.gate_logits && a.gate_mode != 0) gh = 1.f / (1.f + __expf(-a.gate_logits[tok * G + h]));
#pragma unroll 1
      for (int c = 0; c < kD; c += 16) {
        uint32_t v[16];
        tmem_ld16(tO + lane_off + c, v);
        tmem_ld_wait();
        if (!valid) continue;
        float o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float g = gh;
          if (a.gate_logits && a.gate_mode == 0) g = 1.f / (1.f + __expf(-a.gate_logits[tok * G + h * kD + c + i]));
          o[i] = __uint_as_float(v[i]) * inv * g;
        }
        uint4 p0, p1;
        p0.x = pack_bf16x2(o[0], o[1]);
        p0.y = pack_bf16x2(o[2], o[3]);
        p0.z = pack_bf16x2(o[4], o[5]);
        p0.w = pack_bf16x2(o[6], o[7]);
        p1.x = pack_bf16x2(o[8], o[9]);
        p1.y = pack_bf16x2(o[10], o[11]);
        p1.z = pack_bf16x2(o[12], o[13]);
        p1.w = pack_bf16x2(o[14], o[15]);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + tok * HD + h * kD + c);
        dst[0] = p0;
        dst[1] = p1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_prefill_attn_bf16(const PrefillArgs& a, cudaStream_t st) {
  if (a.d_h != kD) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  prof_begin(st, "prefill_attn");
  prefill_attn_kernel<<<dim3(a.q_tiles_per_seq, a.H, a.B), 192, kSmem, st>>>(a);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace gmla
