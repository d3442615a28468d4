// decode_fp8.cuh — absorbed-form decode over an FP8 (E4M3) latent cache
// (included at the end of decode_tc.cu: it shares the split plan and the merge).
//
// The cache holds e4m3 codes c~ with one fp32 scale for the whole cache
// (c = cache_scale * c~), half the bytes of a bf16 cache. The method is that of
// decode_tc.cu ("Gated MLA 计算公式" §一/§二, "精读笔记 03" §5.1, 题4):
//   z_s = q_lat . c_s,  O_lat = sum_s softmax(z)_s c_s,  o = W_v O_lat (gated).
// Both products run on tcgen05 kind::f8f6f4 tensor cores straight from the
// cached codes (no conversion pass):
//   S^T = C~ (Q~)^T   M = 128 tokens, K = 32 latent dims per MMA, N = 2 HG
//   O^T += C~^T P^T   M = 128 latent dims (the cache box read MN-major), K = 32 tokens
// The other operand of each product is not an FP8 quantity of the method, so it
// is carried as a hi + lo pair of e4m3 values (v ~ hi + lo, about 7 significant
// bits): the absorbed query as Q~ = [hi(q_lat / sigma); lo(...)] with one scale
// sigma per (sequence, head), and P' = kPScale p as [hi; lo]. The pair doubles N,
// which costs next to nothing at these widths (an MMA with N <= 64 is bound by
// its A operand). Scores are (S[h] + S[HG + h]) * sigma * cache_scale; the
// weighted sum is (O^T[h] + O^T[HG + h]) * cache_scale / kPScale.
//
// Kernels: decode_absorb_fp8 (q_lat, its scale and hi/lo codes; its last block
// builds the split plan as decode_absorb_plan does), decode_attn_fp8 (below),
// then decode_merge and the W_v GEMM of the bf16 path.
#pragma once
#include <cuda_fp8.h>

namespace gmla {

namespace {
constexpr int kTok = 128;                  // tokens per tile
constexpr int kBox8 = 128 * 128;           // one box: 128 token rows x 128 e4m3 latent dims
constexpr int kNB8 = 4;                    // boxes per tile (d_c = 512)
constexpr int kDc8 = 512;
// The running max of a head is raised only when a tile's max exceeds it by
// more than kRaise8 (log2 units), so p = 2^(s - m) <= 2^kRaise8 and
// P' = kPScale p <= 256, inside E4M3's range (448); weights down to
// 2^-15 stay representable.
constexpr float kRaise8 = 2.f;
constexpr float kPScale = 64.f;

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float from_e4m3(uint8_t c) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}
// hi + lo e4m3 pair of v (hi = e4m3(v), lo = e4m3(v - hi))
__device__ __forceinline__ void split_e4m3(float v, uint8_t& hi, uint8_t& lo) {
  hi = to_e4m3(v);
  lo = to_e4m3(v - from_e4m3(hi));
}
// byte offset of (row, col) in a K-major tile of 128-byte rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_byte(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 4) ^ row) & 7u) << 4) + (col & 15u);
}
}  // namespace

// ---------------------------------------------------------------------------
// absorb: per (head, 8 sequences): q_lat = q_scale * W_k^(h)T q^(h) over all 512
// latent dims, sigma = max |q_lat| / 448, codes hi/lo of q_lat / sigma written to
// the rows of the head's slot; qmul = sigma * cache_scale. The last block runs
// the split plan.
// ---------------------------------------------------------------------------
constexpr int kAbs8B = 8;

__global__ void __launch_bounds__(256) decode_absorb_fp8_kernel(DecodeArgs a) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int n_bblk = (a.B + kAbs8B - 1) / kAbs8B;
  if (static_cast<int>(blockIdx.x) == a.H * n_bblk) {
    griddep_wait();
    decode_plan_block(a);
    return;
  }
  const int h = blockIdx.x / n_bblk;
  const int b0 = (blockIdx.x % n_bblk) * kAbs8B;
  const int nb = min(kAbs8B, a.B - b0);
  const int c0 = threadIdx.x * 2;   // two latent columns per thread
  const __nv_bfloat16* Wk = static_cast<const __nv_bfloat16*>(a.W_k) + static_cast<int64_t>(h) * a.d_h * kDc8;
  __shared__ float sq[kAbs8B][256];
  __shared__ float red[kAbs8B][8];
  __shared__ int s_slot[kAbs8B];
  __shared__ float s_on[kAbs8B];
  griddep_wait();
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const int dq = a.d_h + a.d_rope;
  for (int i = threadIdx.x; i < kAbs8B * a.d_h; i += blockDim.x) {
    const int bi = i / a.d_h, k = i % a.d_h;
    sq[bi][k] = bi < nb ? __bfloat162float(q[(static_cast<int64_t>(b0 + bi) * a.H + h) * dq + k]) : 0.f;
  }
  if (threadIdx.x < kAbs8B) {
    int slot = h;
    float on = 1.f;
    const int bi = threadIdx.x;
    if (a.gate_hard && bi < nb) {
      const float* z = a.gate_logits + static_cast<int64_t>(b0 + bi) * a.H;
      int na = 0;
      slot = head_slot(z, a.H, h, a.gate_mode, a.gate_topk, &na);
      const float gv = head_gate(z, a.H, h, a.gate_mode, a.gate_topk);
      on = gv != 0.f ? 1.f : 0.f;
      a.gvals[static_cast<int64_t>(b0 + bi) * a.H + h] = gv;
      a.head_of_slot[static_cast<int64_t>(b0 + bi) * a.H + slot] = h;
    }
    s_slot[bi] = slot;
    s_on[bi] = on;
  }
  __syncthreads();
  float acc[kAbs8B][2];
#pragma unroll
  for (int bi = 0; bi < kAbs8B; ++bi) acc[bi][0] = acc[bi][1] = 0.f;
  // 16 rows of W_k in flight at a time (the loads, not the FMAs, set the pace)
  constexpr int kRows = 16;
  for (int k0 = 0; k0 < a.d_h; k0 += kRows) {
    __nv_bfloat162 w2[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i)
      w2[i] = k0 + i < a.d_h ? *reinterpret_cast<const __nv_bfloat162*>(Wk + static_cast<int64_t>(k0 + i) * kDc8 + c0)
                             : __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      if (k0 + i >= a.d_h) break;
      const float w0 = __low2float(w2[i]), w1 = __high2float(w2[i]);
#pragma unroll
      for (int bi = 0; bi < kAbs8B; ++bi) {
        acc[bi][0] = fmaf(sq[bi][k0 + i], w0, acc[bi][0]);
        acc[bi][1] = fmaf(sq[bi][k0 + i], w1, acc[bi][1]);
      }
    }
  }
  // per sequence: the largest |q_lat| over the 512 dims (block reduction)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int bi = 0; bi < kAbs8B; ++bi) {
    acc[bi][0] *= a.q_scale;
    acc[bi][1] *= a.q_scale;
    float mx = fmaxf(fabsf(acc[bi][0]), fabsf(acc[bi][1]));
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[bi][warp] = mx;
  }
  __syncthreads();
  uint8_t* qa = static_cast<uint8_t*>(a.qa);
  const int N2 = 2 * a.HG;
  for (int bi = 0; bi < nb; ++bi) {
    float mx = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) mx = fmaxf(mx, red[bi][w]);
    const float sigma = mx > 0.f ? mx / 448.f : 1.f;
    const float inv = 1.f / sigma;
    const int b = b0 + bi, slot = s_slot[bi];
    if (threadIdx.x == 0) a.qmul[static_cast<int64_t>(b) * a.H + slot] = sigma * a.cache_scale * s_on[bi];
    // slots past the launched head groups (heads a top-k gate switches off) are never read
    if (slot >= a.n_hg * a.HG) continue;
    const int64_t row_hi = (static_cast<int64_t>(b) * a.n_hg + slot / a.HG) * N2 + slot % a.HG;
    uint8_t h0, l0, h1, l1;
    split_e4m3(acc[bi][0] * inv * s_on[bi], h0, l0);
    split_e4m3(acc[bi][1] * inv * s_on[bi], h1, l1);
    *reinterpret_cast<uint16_t*>(qa + row_hi * kDc8 + c0) = static_cast<uint16_t>(h0 | (h1 << 8));
    *reinterpret_cast<uint16_t*>(qa + (row_hi + a.HG) * kDc8 + c0) = static_cast<uint16_t>(l0 | (l1 << 8));
  }
}

// ---------------------------------------------------------------------------
// attention over the FP8 cache
// ---------------------------------------------------------------------------
struct Dec8Smem {
  uint64_t full[16], empty[16];   // per ring box
  uint64_t q_full, q_empty, s_full, p_full, o_done, o_free, drain, never;
  uint32_t tmem;
  int abort;
  int vote[3];
  int red[2][4][64];
  float lred[4][64];
  float mfin[64];
};

// 16 heads per CTA: two CTAs share an SM (each holds a ring of 5 boxes, and
// the 256 columns of tensor memory it needs), so one CTA's loads, softmax and
// MMAs overlap the other's; each CTA on its own is bound by the latency of
// that chain, not by bandwidth. 32 heads: one CTA per SM with a deeper ring.
template <int HG>
struct Dec8Cfg {
  static constexpr int kN2 = 2 * HG;                         // hi and lo columns
  static constexpr int kSG = HG >= 32 ? 2 : 1;               // softmax warp groups (head slices)
  static constexpr int kThreads = 64 + 128 * kSG;
  static constexpr int kCtasPerSm = HG == 16 ? 2 : 1;
  static constexpr int kQBytes = kNB8 * kN2 * 128;           // 4 boxes of [2 HG rows x 128 B]
  static constexpr int kPBytes = ((kN2 * 128) + 1023) & ~1023;   // [2 HG rows x 128 tokens]
  static constexpr int kStruct = (static_cast<int>(sizeof(Dec8Smem)) + 127) & ~127;
  static constexpr int kFixed = kQBytes + kPBytes + kStruct + 1024 /*align*/;
  // shared memory of an SM (233472 B) less 1 KB reserved per CTA
  static constexpr int kBudget = kCtasPerSm == 2 ? 233472 / 2 - 1024 : 232448;
  static constexpr int kRingMax = (kBudget - kFixed) / kBox8;
  static constexpr int kRing = kRingMax > 16 ? 16 : kRingMax;
  static constexpr int kSmem = kRing * kBox8 + kFixed;
  static constexpr int kTmemCols = 6 * kN2 <= 256 ? 256 : 512;   // 2 S^T buffers + 4 O^T chunks
  // the next tile's boxes are probed by the parity of their full barrier, which
  // is unambiguous while box c - kRing has been waited for: true up to c =
  // (first box of this tile) + 2 kNB8 - 1 when kRing >= kNB8
  static_assert(kRing >= kNB8 + 1, "the ring holds more than one tile");
  static_assert(kCtasPerSm * kTmemCols <= 512, "tensor memory of the CTAs sharing an SM");
};

template <int HG>
__global__ void __launch_bounds__(64 + 128 * (HG >= 32 ? 2 : 1), (HG == 16 ? 2 : 1))
    decode_attn_fp8_kernel(const __grid_constant__ DecodeArgs a) {
  using C = Dec8Cfg<HG>;
  constexpr int NR = C::kRing, N2 = C::kN2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qs = ring + NR * kBox8;
  uint8_t* pbuf = qs + C::kQBytes;
  Dec8Smem* sm = reinterpret_cast<Dec8Smem*>(pbuf + C::kPBytes);
  volatile int* abort_flag = &sm->abort;

  const int g = blockIdx.x, hg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int heads_valid = min(HG, a.H - hg * HG);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NR; ++i) {
      mbar_init(&sm->full[i], 1);
      mbar_init(&sm->empty[i], 1);
    }
    mbar_init(&sm->q_full, 1);
    mbar_init(&sm->q_empty, 1);
    mbar_init(&sm->s_full, 1);
    mbar_init(&sm->p_full, 128 * C::kSG);
    mbar_init(&sm->o_done, 1);
    mbar_init(&sm->o_free, 128 * C::kSG);
    mbar_init(&sm->drain, 1);
    mbar_init(&sm->never, 1);
    sm->abort = 0;
    sm->vote[0] = sm->vote[1] = sm->vote[2] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();   // the plan, the absorbed queries and the cache rows come from earlier kernels
  const int seg_lo = a.cta_first_seg[g];
  const int seg_hi = (seg_lo < a.cta_first_seg[g + 1]) ? a.cta_first_seg[g + 1] : seg_lo;
  const uint32_t tmem = sm->tmem;
  const uint32_t tO = tmem + 2 * N2;   // O^T chunk j (latent dims 128 j ..) at columns tO + j N2

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&a.cache_map);
      tma_prefetch_desc(&a.qa_map);
    }
    const uint64_t pol_c = a.n_hg > 1 ? l2_evict_normal() : l2_evict_first();
    const uint64_t pol_q = l2_evict_last();
    const bool paged = a.cache.paged != 0;
    const int ps = paged ? a.cache.page_size : kTok;
    uint32_t nbox = 0, nq = 0;
    bool ok = true;
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const int4 sg = a.seg_info[si];
      const int b = sg.x;
      const int L = sg.w;
      if (seg_heads(a, b, hg, heads_valid) == 0) continue;
      if (lane == 0) {
        if (nq > 0 && !mbar_wait(&sm->q_empty, (nq - 1) & 1, abort_flag, a.status)) ok = false;
        if (ok) {
          mbar_arrive_expect_tx(&sm->q_full, C::kQBytes);
          for (int j = 0; j < kNB8; ++j)
            tma_load_2d(&a.qa_map, &sm->q_full, qs + j * N2 * 128, j * 128, (b * a.n_hg + hg) * N2, pol_q);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++nq;
      for (int t = sg.y; t < sg.z && ok; ++t) {
        const int tok0 = t * kTok;
        const int valid = min(kTok, L - tok0);
        const int nchunk = ps >= kTok ? 1 : (valid + ps - 1) / ps;   // <= 16 (page size >= 8)
        int page = 0;
        if (paged && lane < nchunk)
          page = a.cache.block_table[static_cast<int64_t>(b) * a.cache.max_pages_per_seq + (tok0 + lane * ps) / ps];
        const uint32_t tx = ps >= kTok ? kBox8 : nchunk * ps * 128;
        for (int j = 0; j < kNB8; ++j) {
          const uint32_t slot = nbox % NR;
          if (lane == 0) {
            if (nbox >= static_cast<uint32_t>(NR) &&
                !mbar_wait(&sm->empty[slot], ((nbox / NR) & 1) ^ 1, abort_flag, a.status))
              ok = false;
            if (ok) mbar_arrive_expect_tx(&sm->full[slot], tx);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          uint8_t* dst = ring + slot * kBox8;
          if (!paged) {
            if (lane == 0) tma_load_2d(&a.cache_map, &sm->full[slot], dst, j * 128, b * a.cache.capacity + tok0, pol_c);
          } else if (ps >= kTok) {
            if (lane == 0) tma_load_3d(&a.cache_map, &sm->full[slot], dst, j * 128, tok0 % ps, page, pol_c);
          } else if (lane < nchunk) {
            tma_load_3d(&a.cache_map, &sm->full[slot], dst + lane * ps * 128, j * 128, 0, page, pol_c);
          }
          ++nbox;
        }
      }
    }
    if (lane == 0 && *abort_flag) {   // let issued copies land before the block exits
      for (uint32_t c = nbox > static_cast<uint32_t>(NR) ? nbox - NR : 0; c < nbox; ++c)
        mbar_drain(&sm->full[c % NR], (c / NR) & 1);
      if (nq) mbar_drain(&sm->q_full, (nq - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_e4m3_f32(128, N2, false, false);
      constexpr uint32_t idO = idesc_e4m3_f32(128, N2, true, false);
      const uint32_t ring_a = smem_u32(ring), q_a = smem_u32(qs), p_a = smem_u32(pbuf);
      const uint64_t dRing = sdesc_sw128(ring_a, 16, 1024), dQ = sdesc_sw128(q_a, 16, 1024);
      const uint64_t dRingMN = sdesc_sw128(ring_a, kBox8, 1024);   // a box read as [tokens (K) x 128 latent dims (M)]
      const uint64_t dP = sdesc_sw128(p_a, 16, 1024);
      auto s_box = [&](uint32_t c, int j, uint32_t tSb) {   // S^T += box j of the tile x its Q box
        const uint64_t da = dRing + (c % NR) * (kBox8 / 16);
        const uint64_t db = dQ + j * (N2 * 128 / 16);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_f8(tSb, da + kk * 2, db + kk * 2, idS, (j | kk) != 0);
      };
      uint32_t nbox = 0, ntile = 0, nseg = 0;
      int early = 0;
      bool ok = true;
      if (a.test_stall && g == 0 && hg == 0) ok = mbar_wait(&sm->never, 0, abort_flag, a.status);
      for (int si = seg_lo; si < seg_hi && ok; ++si) {
        const int4 sg = a.seg_info[si];
        if (seg_heads(a, sg.x, hg, heads_valid) == 0) continue;
        if (!mbar_wait(&sm->q_full, nseg & 1, abort_flag, a.status)) { ok = false; break; }
        for (int t = sg.y; t < sg.z; ++t, ++ntile) {
          const uint32_t tSb = tmem + (ntile & 1) * N2;
          for (int j = early; j < kNB8; ++j) {
            const uint32_t c = nbox + j;
            if (!mbar_wait(&sm->full[c % NR], (c / NR) & 1, abort_flag, a.status)) { ok = false; break; }
            s_box(c, j, tSb);
          }
          if (!ok) break;
          if (t + 1 == sg.z) umma_commit(&sm->q_empty);
          umma_commit(&sm->s_full);
          // the next tile's boxes that have landed (a non-blocking probe)
          early = 0;
          if (t + 1 < sg.z) {
            const uint32_t tSn = tmem + ((ntile + 1) & 1) * N2;
            for (int j = 0; j < kNB8; ++j) {
              const uint32_t c = nbox + kNB8 + j;
              if (!mbar_test(&sm->full[c % NR], (c / NR) & 1)) break;
              s_box(c, j, tSn);
              ++early;
            }
          }
          if (!mbar_wait(&sm->p_full, ntile & 1, abort_flag, a.status)) { ok = false; break; }
          const bool first = (t == sg.y);
          if (first && nseg > 0 && !mbar_wait(&sm->o_free, (nseg - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int j = 0; j < kNB8; ++j) {
            const uint32_t slot = (nbox + j) % NR;
            const uint64_t da = dRingMN + slot * (kBox8 / 16);
#pragma unroll
            for (int kk = 0; kk < kTok / 32; ++kk)
              umma_f8(tO + j * N2, da + kk * (4096 / 16), dP + kk * 2, idO, (!first || kk > 0) ? 1u : 0u);
            umma_commit(&sm->empty[slot]);
          }
          nbox += kNB8;
        }
        if (!ok) break;
        umma_commit(&sm->o_done);
        ++nseg;
      }
      if (!ok) {
        umma_commit(&sm->drain);
        mbar_drain(&sm->drain, 0);
      }
    }
  } else {
    // ------------------------------ softmax warps ------------------------------
    constexpr int SG = C::kSG, HT = HG / SG;
    const int q4 = warp & 3;
    const int h0 = SG == 1 ? 0 : ((warp - 2) >> 2) * HT;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int ltid = threadIdx.x - 64;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float o_mul = a.cache_scale / kPScale;
    uint32_t nbox = 0, ntile = 0, nseg = 0;
    bool ok = true;
    for (int si = seg_lo; si < seg_hi; ++si) {
      const int4 sg = a.seg_info[si];
      const int b = sg.x;
      const int L = sg.w;
      const int S0 = a.seq_starts ? a.seq_starts[b] : 0;
      const int hv = seg_heads(a, b, hg, heads_valid);
      if (hv == 0) continue;
      float mul[HT], m[HT], lsum[HT];
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        const int slot = hg * HG + h0 + h;
        mul[h] = (h0 + h < hv && slot < a.H) ? a.qmul[static_cast<int64_t>(b) * a.H + slot] : 0.f;
        m[h] = NEG_INF;
        lsum[h] = 0.f;
      }
      for (int t = sg.y; t < sg.z; ++t, ++ntile) {
        const bool first = (t == sg.y);
        ok = ok && mbar_wait(&sm->s_full, ntile & 1, abort_flag, a.status);
        tc_fence_after();
        const uint32_t tS = tmem + (ntile & 1) * N2 + lane_off + h0;
        const int valid = min(kTok, L - t * kTok);
        const bool rv = row < valid && t * kTok + row >= S0;
        auto load16 = [&](int c, float (&x)[16]) {   // score = (hi + lo) * sigma * cache_scale
          uint32_t vh[16], vl[16];
          tmem_ld16(tS + c, vh);
          tmem_ld16(tS + HG + c, vl);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            x[j] = rv ? (__uint_as_float(vh[j]) + __uint_as_float(vl[j])) * mul[c + j] : NEG_INF;
        };
        bool need = first;
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          float x[16];
          load16(c, x);
#pragma unroll
          for (int j = 0; j < 16; ++j) need |= x[j] > m[c + j] + kRaise8;
        }
        const int par = ntile & 1;
        const int vslot = static_cast<int>(ntile % 3u);
        if (__any_sync(0xffffffffu, need) && lane == 0) atomicOr(&sm->vote[vslot], 1);
        asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");
        const bool need_all = sm->vote[vslot] != 0;
        if (ltid == 0) sm->vote[(vslot + 2) % 3] = 0;
        if (need_all) {
#pragma unroll
          for (int c = 0; c < HT; c += 16) {
            float x[16];
            load16(c, x);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int k = __reduce_max_sync(0xffffffffu, float_to_ordered(x[j]));
              if (lane == 0) sm->red[par][q4][h0 + c + j] = k;
            }
          }
          asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");
#pragma unroll
          for (int c = 0; c < HT; c += 16) {
            float alpha[16];
            bool rescale = false;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int h = c + j;
              int k = sm->red[par][0][h0 + h];
              k = max(k, sm->red[par][1][h0 + h]);
              k = max(k, sm->red[par][2][h0 + h]);
              k = max(k, sm->red[par][3][h0 + h]);
              const float tmax = ordered_to_float(k);
              const float mn = fmaxf(m[h], tmax);
              alpha[j] = (m[h] == NEG_INF) ? 0.f : ex2_approx(m[h] - mn);
              rescale |= (mn > m[h]) && !first;
              m[h] = mn;
              lsum[h] *= alpha[j];
            }
            if (rescale) {   // the hi and lo columns of O^T of these heads scale by alpha
#pragma unroll 1
              for (int mc = 0; mc < kNB8; ++mc) {
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                  uint32_t v[16];
                  const uint32_t col = tO + lane_off + mc * N2 + part * HG + h0 + c;
                  tmem_ld16(col, v);
                  tmem_ld_wait();
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha[j]);
                  tmem_st16(col, v);
                }
              }
              tmem_st_wait();
            }
          }
        }
        // P' = kPScale exp2(s - m) as a hi + lo e4m3 pair, this thread's token column
        // of P [2 HG heads x 128 tokens] (K-major, 128-byte swizzle)
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          float x[16];
          load16(c, x);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int h = h0 + c + j;
            const float p = rv ? ex2_approx(x[j] - m[c + j]) : 0.f;
            lsum[c + j] += p;
            uint8_t hi, lo;
            split_e4m3(p * kPScale, hi, lo);
            pbuf[sw128_byte(h, row)] = hi;
            pbuf[sw128_byte(HG + h, row)] = lo;
          }
        }
        if (!rv) {   // rows outside [start, L) may hold anything (a NaN code): zero them
#pragma unroll 1
          for (int j = h0 / HT; j < kNB8; j += SG) {
            uint8_t* box = ring + ((nbox + j) % NR) * kBox8 + row * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) reinterpret_cast<uint4*>(box)[k] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm->p_full);
        nbox += kNB8;
      }
      // ---- segment end: the partial (O, m, l)
      ok = ok && mbar_wait(&sm->o_done, nseg & 1, abort_flag, a.status);
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        float v = lsum[h];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) sm->lred[q4][h0 + h] = v;
        if (SG > 1 && lane == 0 && q4 == 0) sm->mfin[h0 + h] = m[h];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");
      const int64_t pbase = (static_cast<int64_t>(hg) * a.max_seg + si) * HG;
      if (ok && ltid < hv) {
        float l = 0.f, mh = NEG_INF;
        if (SG == 1) {
#pragma unroll
          for (int h = 0; h < HT; ++h)
            if (h == ltid) mh = m[h];
        } else {
          mh = sm->mfin[ltid];
        }
        for (int w = 0; w < 4; ++w) l += sm->lred[w][ltid];
        a.ml_part[(pbase + ltid) * 2 + 0] = mh;
        a.ml_part[(pbase + ltid) * 2 + 1] = l;
      }
#pragma unroll 1
      for (int mc = 0; mc < kNB8; ++mc) {
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          uint32_t vh[16], vl[16];
          tmem_ld16(tO + lane_off + mc * N2 + h0 + c, vh);
          tmem_ld16(tO + lane_off + mc * N2 + HG + h0 + c, vl);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (ok && h0 + c + j < hv)
              a.o_part[(pbase + h0 + c + j) * kDc8 + mc * 128 + row] =
                  (__uint_as_float(vh[j]) + __uint_as_float(vl[j])) * o_mul;
          }
        }
      }
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");
      mbar_arrive(&sm->o_free);
      ++nseg;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int HG>
static cudaError_t launch_attn_fp8(const DecodeArgs& a, cudaStream_t st) {
  using C = Dec8Cfg<HG>;
  auto k = decode_attn_fp8_kernel<HG>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  prof_begin(st, "decode_attn");
  e = launch_pdl(k, dim3(a.G, a.n_hg), dim3(C::kThreads), C::kSmem, st, 1, a);
  prof_end(st);
  return e;
}

}  // namespace gmla
