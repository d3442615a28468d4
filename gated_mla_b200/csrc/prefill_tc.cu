// prefill_tc.cu — causal attention of whole prompts on tcgen05 tensor cores,
// explicit form ("Gated MLA 计算公式" §一/§二): K^(h), V^(h) were rebuilt from the
// cached latents by the GEMM of gemm_tc.cu; here
//   S = Q K^T (TMEM, fp32)  ->  online softmax over keys s <= t (fp32)
//   O += P V (TMEM, fp32)   ->  o = O / l, gated by sigmoid(g) on the way out.
//
// One CTA per (pair of 128-query tiles, head, sequence). The two query tiles
// A (rows 256 i ..) and B (rows 256 i + 128 ..) share every K/V tile that TMA
// brings in, and they take turns on the tensor cores: while the softmax warps
// of A turn S_A(j) into P, the MMA warp runs S_B(j) and O_B(j-1), and the
// other way round. Each tile keeps S and O in tensor memory (128 + 128
// columns); the softmax writes P (bf16) over the first half of S's columns
// and the P V product reads it from there as the A operand, so P never goes
// through shared memory.
// Roles: warp 0 TMA, one thread of warp 1 the MMAs, warps 2..5 the softmax
// and epilogue of tile A (one query row per thread), warps 6..9 those of B.
// The running max of a row is raised only when a tile's max exceeds it by
// more than 2^8 (the final normalisation uses the same reference, so the
// result is exact); O is rescaled in TMEM only then.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gmla {

namespace {
constexpr int kBQ = 128;          // queries per tile
constexpr int kBK = 128;          // keys per tile
constexpr int kD = 128;           // head dim
constexpr int kDR = 64;           // decoupled RoPE dims (one box) when present
constexpr int kBox = 128 * 128;   // one [128 rows x 64] bf16 box: 16 KB
constexpr int kTile = 2 * kBox;   // [128 rows x 128] bf16
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;   // per tile: S/P 128 columns + O 128 columns

// NoPE: two query tiles per CTA, Q and K rows of d_h = 128 (2 boxes).
// Decoupled RoPE: each Q and K row grows by the 64 rotated dims (a third box:
// q^R of the head; k^R shared by all heads, read from the cache rows), and one
// query tile per CTA keeps the stages in shared memory.
template <bool kRope>
struct PfCfg {
  static constexpr int kQKBoxes = kRope ? 3 : 2;
  static constexpr int kQTile = kQKBoxes * kBox;
  static constexpr int kKTile = kQKBoxes * kBox;
  static constexpr int kQTiles = kRope ? 1 : 2;
  static constexpr int kSmem = kQTiles * kQTile + kStages * (kKTile + kTile) + 1024 + 256;
};

struct PfBars {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain;
  uint32_t tmem;
  int abort;
};
}  // namespace

template <bool kRope>
__global__ void __launch_bounds__(320, 1) prefill_attn_kernel(const __grid_constant__ PrefillArgs a) {
  using C = PfCfg<kRope>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                             // [tile A, tile B]
  uint8_t* sK = sQ + C::kQTiles * C::kQTile;      // [stage]
  uint8_t* sV = sK + kStages * C::kKTile;         // [stage]
  PfBars* bars = reinterpret_cast<PfBars*>(sV + kStages * kTile);
  volatile int* abort_flag = &bars->abort;

  griddep_wait();   // Q, K and V come from the kernels before this one
  const int b = blockIdx.z, h = blockIdx.y;
  const int beg = a.cu_seqlens[b];
  const int len = a.cu_seqlens[b + 1] - beg;
  const int n_qt = (len + kBQ - 1) / kBQ;
  // NoPE: a pair of query tiles per CTA; RoPE: one (tile B absent)
  const int pair = (kRope ? n_qt : (n_qt + 1) / 2) - 1 - static_cast<int>(blockIdx.x);   // long rows first
  if (pair < 0) return;
  const int qtA = kRope ? pair : 2 * pair, qtB = qtA + 1;
  const bool hasB = !kRope && qtB < n_qt;
  const int n_kv = hasB ? qtB + 1 : qtA + 1;     // causal: key tiles 0..last query tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dq = a.d_h + (kRope ? kDR : 0);      // q row of a head: [q | q^R]

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_done[i], 1);
    }
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
  // tile X: S/P at columns [256 X, 256 X + 128), O at [256 X + 128, 256 X + 256)

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.q_map);
      tma_prefetch_desc(&a.k_map);
      tma_prefetch_desc(&a.v_map);
      const uint64_t pol = l2_evict_last();
      mbar_arrive_expect_tx(&bars->q_full, (hasB ? 2 : 1) * C::kQTile);
      for (int x = 0; x < (hasB ? 2 : 1); ++x)
        for (int kb = 0; kb < C::kQKBoxes; ++kb)
          tma_load_2d(&a.q_map, &bars->q_full, sQ + x * C::kQTile + kb * kBox, h * dq + kb * 64,
                      beg + (qtA + x) * kBQ, pol);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&bars->kv_empty[st], ((j / kStages) & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(&bars->kv_full[st], C::kKTile + kTile);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_2d(&a.k_map, &bars->kv_full[st], sK + st * C::kKTile + kb * kBox, h * kD + kb * 64,
                      beg + j * kBK, pol);
          tma_load_2d(&a.v_map, &bars->kv_full[st], sV + st * kTile + kb * kBox, h * kD + kb * 64,
                      beg + j * kBK, pol);
        }
        // k^R of these keys (rotated, shared by all heads): the RoPE columns of the cache rows
        if (kRope)
          tma_load_2d(&a.kr_map, &bars->kv_full[st], sK + st * C::kKTile + 2 * kBox, a.d_c,
                      b * a.cache_capacity + j * kBK, pol);
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
      constexpr uint32_t idO = idesc_bf16_f32(128, 128, false, true);    // P from TMEM, V MN-major
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      auto issue_s = [&](int x, int j) {   // S_x = Q_x K_j^T (+ Q^R_x K^R_j^T)
        const uint32_t kbase = ka + (j % kStages) * C::kKTile, qbase = qa + x * C::kQTile;
#pragma unroll
        for (int k = 0; k < C::kQKBoxes * 4; ++k) {
          const int kb = k >> 2, kk = k & 3;
          umma_bf16(tmem + 256 * x, sdesc_sw128(qbase + kb * kBox + kk * 32, 16, 1024),
                    sdesc_sw128(kbase + kb * kBox + kk * 32, 16, 1024), idS, k != 0);
        }
        umma_commit(&bars->s_full[x]);
      };
      auto issue_o = [&](int x, int j) {   // O_x += P_x V_j, P read from the S columns
        const uint32_t vbase = va + (j % kStages) * kTile;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16_ta(tmem + 256 * x + 128, tmem + 256 * x + k * 8,
                       sdesc_sw128(vbase + k * 2048, kBox, 1024), idO, (j > 0 || k > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.status) &&
                mbar_wait(&bars->kv_full[0], 0, abort_flag, a.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (hasB) issue_s(1, 0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const bool nextkv = j + 1 < n_kv;
        bool next_loaded = false;
        if (j <= qtA) {
          if (!mbar_wait(&bars->p_full[0], j & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          issue_o(0, j);
          if (j == qtA) umma_commit(&bars->o_done[0]);   // tile A's epilogue overlaps B's last step
          if (j + 1 <= qtA) {
            if (!mbar_wait(&bars->kv_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            next_loaded = true;
            issue_s(0, j + 1);   // K tile ordered by its TMA barrier; TMEM reuse by the P_A wait
          }
        }
        if (hasB) {
          if (!mbar_wait(&bars->p_full[1], j & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          issue_o(1, j);
        }
        umma_commit(&bars->kv_empty[j % kStages]);
        if (hasB && nextkv) {
          if (!next_loaded &&
              !mbar_wait(&bars->kv_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          issue_s(1, j + 1);   // TMEM reuse ordered by the P_B wait above
        }
      }
      if (ok) {
        umma_commit(&bars->o_done[1]);
      } else {
        umma_commit(&bars->drain);
        mbar_drain(&bars->drain, 0);
      }
    }
  } else {
    // ------------------------- softmax + epilogue of one tile -------------------------
    // Four warps per tile, one query row per thread: 128 keys per tile step and
    // 128 output columns at the end.
    const int x = warp < 6 ? 0 : 1;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // query row in the tile
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tS = tmem + 256 * x + lane_off, tO = tS + 128;
    const int qt = x == 0 ? qtA : qtB;
    const int qi = qt * kBQ + r;                  // position in the sequence
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m = NEG_INF, l = 0.f;
    bool ok = true;
    const bool active = x == 0 || hasB;
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    // P = exp2(s*scale - m) for 32 keys [k0, k0 + 32) as 16 bf16 pairs, stored
    // over S at columns [k0/2, k0/2 + 16); returns the sum of the 32 values
    auto p_chunk = [&](const uint32_t (&u)[32], int k0, bool diag, uint64_t nm2) -> uint64_t {
      uint32_t pk[16];
      uint64_t ls2[2] = {0ull, 0ull};
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float x0, x1, p0, p1;
        f2_unpack(ffma2(f2_pack(__uint_as_float(u[i]), __uint_as_float(u[i + 1])), sc2, nm2), x0, x1);
        if ((i & 2) == 0) {   // half the exponentials on the special-function unit,
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        } else {              // half on the FMA pipes
          exp2_poly2(x0, x1, p0, p1);
        }
        if (diag) {
          p0 = (k0 + i <= r) ? p0 : 0.f;
          p1 = (k0 + i + 1 <= r) ? p1 : 0.f;
        }
        ls2[(i >> 1) & 1] = fadd2(ls2[(i >> 1) & 1], f2_pack(p0, p1));
        pk[i >> 1] = pack_bf16x2(p0, p1);
      }
      tmem_st16(tS + (k0 >> 1), pk);
      return fadd2(ls2[0], ls2[1]);
    };
    for (int j = 0; active && j <= qt; ++j) {
      if (j == max(0, qt - 4) && a.gate_logits && qi < len) {
        // this row's gate logits, needed by the epilogue, requested into L2 now
        const int G = a.gate_mode == 0 ? a.H * kD : a.H;
        const float* gr = a.gate_logits + static_cast<int64_t>(beg + qi) * G + (a.gate_mode == 0 ? h * kD : h);
#pragma unroll
        for (int c = 0; c < (a.gate_mode == 0 ? 4 : 1); ++c) prefetch_l2(gr + c * 32);
      }
      ok = ok && mbar_wait(&bars->s_full[x], j & 1, abort_flag, a.status);
      tc_fence_after();
      const bool diag = (j == qt);
      // the row max of the raw scores (the scale is positive): keys 64..127 are
      // read while keys 0..63 are scanned
      float pm[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) pm[k] = NEG_INF;
      {
        uint32_t c0[32], c1[32], c2[32], c3[32];
        tmem_ld32(tS, c0);
        tmem_ld32(tS + 32, c1);
        tmem_ld_wait_regs(c0);
        tmem_ld_wait_regs(c1);
        tmem_ld32(tS + 64, c2);
        tmem_ld32(tS + 96, c3);
        if (!diag) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            pm[0] = fmax3(pm[0], __uint_as_float(c0[i]), __uint_as_float(c0[i + 1]));
            pm[1] = fmax3(pm[1], __uint_as_float(c1[i]), __uint_as_float(c1[i + 1]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i <= r) pm[0] = fmaxf(pm[0], __uint_as_float(c0[i]));
            if (32 + i <= r) pm[1] = fmaxf(pm[1], __uint_as_float(c1[i]));
          }
        }
        tmem_ld_wait_regs(c2);
        tmem_ld_wait_regs(c3);
        if (!diag) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            pm[2] = fmax3(pm[2], __uint_as_float(c2[i]), __uint_as_float(c2[i + 1]));
            pm[3] = fmax3(pm[3], __uint_as_float(c3[i]), __uint_as_float(c3[i + 1]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (64 + i <= r) pm[2] = fmaxf(pm[2], __uint_as_float(c2[i]));
            if (96 + i <= r) pm[3] = fmaxf(pm[3], __uint_as_float(c3[i]));
          }
        }
      }
      const float tmax = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) * a.scale_log2;
      float alpha = 1.f;
      if (j == 0 || tmax > m + 8.f) {
        const float mn = fmaxf(m, tmax);
        alpha = (m == NEG_INF) ? 0.f : ex2_approx(m - mn);
        l *= alpha;
        m = mn;
      }
      // The raise is decided per row, but the TMEM loads and stores are
      // warp-collective: when any row of the warp raised its max, the whole warp
      // rescales its O rows, the others by 1. O of the previous tile is complete
      // here: S of this tile was issued after it.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          uint32_t w[16];
          tmem_ld16(tO + c, w);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) w[k] = __float_as_uint(__uint_as_float(w[k]) * alpha);
          tmem_st16(tO + c, w);
        }
        tmem_st_wait();
      }
      // P over S, 32 keys at a time, the next chunk's scores read while this chunk's
      // P is computed (P of a chunk only overwrites columns already read)
      const uint64_t nm2 = f2_pack(-m, -m);
      uint64_t ls = 0ull;
      {
        uint32_t ua[32], ub[32];
        tmem_ld32(tS, ua);
        tmem_ld_wait_regs(ua);
        tmem_ld32(tS + 32, ub);
        ls = fadd2(ls, p_chunk(ua, 0, diag, nm2));
        tmem_ld_wait_regs(ub);
        tmem_ld32(tS + 64, ua);
        ls = fadd2(ls, p_chunk(ub, 32, diag, nm2));
        tmem_ld_wait_regs(ua);
        tmem_ld32(tS + 96, ub);
        ls = fadd2(ls, p_chunk(ua, 64, diag, nm2));
        tmem_ld_wait_regs(ub);
        ls = fadd2(ls, p_chunk(ub, 96, diag, nm2));
      }
      {
        float s0, s1;
        f2_unpack(ls, s0, s1);
        l += s0 + s1;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[x]);
    }
    // warp-uniform decision: the epilogue's TMEM loads are warp-collective
    bool epi = active && ok && mbar_wait(&bars->o_done[x], 0, abort_flag, a.status);
    epi = __all_sync(0xffffffffu, epi);
    if (epi) {
      tc_fence_after();
      const bool valid = qi < len;
      const int HD = a.H * kD;
      const int G = a.gate_mode == 0 ? HD : a.H;
      const int64_t tok = beg + qi;
      const float inv = 1.f / l;
      float gh = 1.f;
      if (valid && a.gate_logits && a.gate_mode != 0)
        gh = gate_is_hard(a.gate_mode) ? head_gate(a.gate_logits + tok * G, a.H, h, a.gate_mode, a.gate_topk)
                                       : __fdividef(1.f, 1.f + __expf(-__ldg(a.gate_logits + tok * G + h)));
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        // the gate logits first, so their latency overlaps the TMEM read
        float g[32];
        if (valid && a.gate_logits && a.gate_mode == 0) {
          const float4* gp = reinterpret_cast<const float4*>(a.gate_logits + tok * G + h * kD + c);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 q4v = __ldg(gp + i);
            g[4 * i] = q4v.x;
            g[4 * i + 1] = q4v.y;
            g[4 * i + 2] = q4v.z;
            g[4 * i + 3] = q4v.w;
          }
        }
        uint32_t w[32];
        tmem_ld32(tO + c, w);
        tmem_ld_wait();
        if (!valid) continue;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + tok * HD + h * kD + c);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float o[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float gk = a.gate_mode == 0 && a.gate_logits ? sigmoid_tanh(g[i + k]) : gh;
            o[k] = __uint_as_float(w[i + k]) * inv * gk;
          }
          uint4 pk;
          pk.x = pack_bf16x2(o[0], o[1]);
          pk.y = pack_bf16x2(o[2], o[3]);
          pk.z = pack_bf16x2(o[4], o[5]);
          pk.w = pack_bf16x2(o[6], o[7]);
          dst[i >> 3] = pk;
        }
      }
    }
  }

  // one lane of a warp ran a role alone: reconverge before the block-wide barrier
  // (a partly arrived warp must not count as arrived)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool kRope>
static cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st) {
  using C = PfCfg<kRope>;
  auto k = prefill_attn_kernel<kRope>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int ctas = kRope ? a.q_tiles_per_seq : (a.q_tiles_per_seq + 1) / 2;
  prof_begin(st, "prefill_attn");
  e = launch_pdl(k, dim3(ctas, a.H, a.B), dim3(320), C::kSmem, st, 1, a);
  prof_end(st);
  return e;
}

cudaError_t launch_prefill_attn_bf16(const PrefillArgs& a, cudaStream_t st) {
  if (a.d_h != kD || (a.d_rope != 0 && a.d_rope != kDR)) return cudaErrorInvalidValue;
  return a.d_rope ? launch_prefill<true>(a, st) : launch_prefill<false>(a, st);
}

}  // namespace gmla
