// decode_tc.cu — absorbed-form Gated MLA decode on tcgen05 tensor cores.
//
// The method ("Gated MLA 计算公式" §一/§二, "精读笔记 03" §5.1, §5.2, 题4):
//   q_lat^(h) = W_k^(h)T q^(h)                      (absorption of W_k into the query)
//   z_s       = scale * (q_lat^(h) . c_s + q^R(h) . k^R_s),   s < L
//   O_lat     = sum_s softmax(z)_s c_s              (weighted sum in latent space)
//   o^(h)     = W_v^(h) O_lat;   out = sigmoid(g) ⊙ o   (W_v absorbed on the output side)
//
// Kernels, in launch order (the W_v product with the gate is a GEMM of gemm_tc.cu):
//   1. decode_absorb_tc q_lat = W_k^T q (times scale*log2 e) on tcgen05, bf16, with
//                       q^R appended; its last block splits the cached tokens of all
//                       sequences into equal per-CTA ranges of 128-token tiles
//                       (segments).
//   2. decode_attn      per (CTA range, head group of HG heads): TMA streams the
//                       latent rows through a ring of 16 KB boxes (128 tokens x 64
//                       latent dims) in pairs, one full and one empty barrier per
//                       pair; tcgen05 computes S^T = C Q_lat^T (M = 128 tokens,
//                       N = HG) into one of two TMEM buffers; the softmax warps (four,
//                       or eight as two head slices when HG >= 32) turn S^T into P
//                       (online softmax in fp32, rescaling only when a running max
//                       grows by > 2^8) and store P MN-major in shared memory;
//                       tcgen05 accumulates O^T = C^T P^T (M = 128 latent dims,
//                       N = HG) in TMEM. While the softmax works on a tile, the MMA
//                       warp issues the score MMAs of the next tile's pairs that have
//                       landed. At a segment end the partial (O, m, l) goes out.
//   3. decode_merge     merges the partials of each (sequence, head) by their
//                       log-sum-exp weights into O_lat (bf16 [H, B, d_c]), which the
//                       W_v GEMM turns into the gated head outputs.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gmla {

constexpr int kTileTok = 128;   // tokens per tile (MMA M of S^T)
constexpr int kBoxBytes = 128 * 128;   // one box: 128 token rows x 64 bf16
constexpr int kDc = 512;        // latent width handled by the tensor-core path
constexpr int kNcBox = kDc / 64;

// ---------------------------------------------------------------------------
// 1. plan
// ---------------------------------------------------------------------------
// Exclusive prefix sum over the block (blockDim a multiple of 32); *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) s_warp[w] = inc;
  __syncthreads();
  if (w == 0) {
    const int x = lane < static_cast<int>(blockDim.x >> 5) ? s_warp[lane] : 0;
    int y = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += n;
    }
    s_warp[lane] = y - x;
    if (lane == 31) *total = y;
  }
  __syncthreads();
  const int r = s_warp[w] + inc - v;
  __syncthreads();
  return r;
}

// 128-token tiles that cover positions [start, L) of a sequence.
__device__ __forceinline__ int seq_tiles(int L, int start) {
  return L > start ? (L + kTileTok - 1) / kTileTok - start / kTileTok : 0;
}

// Tiles of 128 tokens of all sequences, concatenated, are cut into G equal
// ranges (one per CTA of a head group). A segment is the part of one sequence
// inside one range; seg_info = {sequence, first tile, end tile, sequence length}
// (the length carried along saves the attention kernel a dependent load).
// A CTA pays about one to two tiles' time for each segment it starts (the
// partial of the previous one written, the next absorbed queries loaded; more
// tiles' worth where tiles are cheap, as with the FP8 cache). So when the CTAs
// average at least 4 tiles, each sequence's range is preceded by two virtual
// tiles: a range that crosses a sequence start holds two real tiles fewer.
// (Ranges then span >= 4 units and the virtual runs 2, each followed by a real
// tile, so every range still holds a real tile.)
__device__ void decode_plan_block(const DecodeArgs& a) {
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ int s_sum, s_nz;
  const int tid = threadIdx.x;
  const int limit = a.cache.paged ? a.cache.max_pages_per_seq * a.cache.page_size : a.cache.capacity;
  if (tid == 0) s_sum = s_nz = 0;
  __syncthreads();
  for (int b = tid; b < a.B; b += blockDim.x) {
    int L = a.seq_lens[b];
    const int s0 = a.seq_starts ? a.seq_starts[b] : 0;
    if (L < 0 || L > limit || b >= a.cache.batch || s0 < 0) {
      report_status(a.status, kStatusRange);
      L = 0;
    }
    const int t = seq_tiles(L, s0);
    atomicAdd(&s_sum, t);
    if (t > 0) atomicAdd(&s_nz, 1);
  }
  __syncthreads();
  const int total = s_sum;
  const int vu = total >= 4 * a.G ? 2 : 0;        // virtual units before each sequence with tiles
  const int total_u = total + vu * s_nz;
  const int tpc = total_u > 0 ? (total_u + a.G - 1) / a.G : 1;
  int unit_carry = 0, seg_carry = 0;
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int b = base + tid;
    int L = b < a.B ? a.seq_lens[b] : 0;
    const int s0 = (b < a.B && a.seq_starts) ? a.seq_starts[b] : 0;
    if (L < 0 || L > limit || b >= a.cache.batch || s0 < 0) L = 0;
    const int t = seq_tiles(L, s0);
    const int ts = s0 / kTileTok;   // first tile of the sequence's range
    int usum, ssum;
    const int P = unit_carry + block_excl_scan(t > 0 ? t + vu : 0, s_warp, &s_total);   // first unit
    usum = s_total;
    const int Q = P + vu;           // unit of the sequence's first tile
    int nseg = 0, g_first = 0;
    if (t > 0) {
      g_first = Q / tpc;
      nseg = (Q + t - 1) / tpc - g_first + 1;
    }
    const int S = seg_carry + block_excl_scan(nseg, s_warp, &s_total);
    ssum = s_total;
    if (b < a.B) {
      a.seq_first_seg[b] = S;
      for (int k = 0; k < nseg; ++k) {
        const int g = g_first + k;
        const int lo = max(Q, g * tpc), hi = min(Q + t, (g + 1) * tpc);
        a.seg_info[S + k] = make_int4(b, ts + lo - Q, ts + hi - Q, L);
        if (g * tpc >= P) a.cta_first_seg[g] = S + k;   // range g starts inside sequence b's units
      }
    }
    unit_carry += usum;
    seg_carry += ssum;
  }
  if (tid == 0) a.seq_first_seg[a.B] = seg_carry;
  const int g_used = total_u > 0 ? (total_u - 1) / tpc + 1 : 0;
  for (int g = g_used + tid; g <= a.G; g += blockDim.x) a.cta_first_seg[g] = seg_carry;
  if (a.gate_hard) {   // heads of each sequence whose gate is not 0
    for (int b = tid; b < a.B; b += blockDim.x) {
      int na = 0;
      head_slot(a.gate_logits + static_cast<int64_t>(b) * a.H, a.H, 0, a.gate_mode, a.gate_topk, &na);
      a.n_act[b] = na;
    }
  }
}

// ---------------------------------------------------------------------------
// 2. absorb: qa[b, h, :d_c] = bf16(q_scale * W_k^(h)T q^(h)), qa[b, h, d_c:] = bf16(q_scale * q^R)
//    On tcgen05, one CTA per (head, 128 latent columns, chunk of up to 128
//    sequences): q_lat^T = W_k^(h)T q^T with M = 128 latent columns (A = W_k^(h),
//    MN-major: its rows are d_h, latent columns contiguous), N = sequences (B = q,
//    K-major), K = d_h, the accumulator in TMEM. W_k is a weight that no kernel
//    writes, so its boxes are requested before waiting for the queries. The last
//    CTA of the grid runs the split plan instead.
// ---------------------------------------------------------------------------
constexpr int kAbsorbM = 128;     // latent columns per CTA

struct AbsorbSmem {
  uint64_t full, mma_done;
  uint32_t tmem;
  int abort;
  int slot[128];
  float on[128];
};

size_t absorb_smem_bytes(int d_h, int bn) {
  return static_cast<size_t>(2 * d_h * 128 + (d_h / 64) * bn * 128) + 1024 + sizeof(AbsorbSmem);
}

__global__ void __launch_bounds__(128) decode_absorb_tc_kernel(const __grid_constant__ DecodeArgs a) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int n_ct = a.d_c / kAbsorbM;
  if (static_cast<int>(blockIdx.x) == a.H * n_ct) {
    if (blockIdx.y == 0) {
      griddep_wait();
      decode_plan_block(a);
    }
    return;
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int BN = a.absorb_bn;
  const int nkb = a.d_h / 64;
  uint8_t* sA = smem;                                  // 2 boxes [d_h rows][64 latent columns]
  uint8_t* sB = sA + 2 * a.d_h * 128;                  // nkb boxes [BN sequences][64 of d_h]
  AbsorbSmem* sm = reinterpret_cast<AbsorbSmem*>(sB + nkb * BN * 128);
  volatile int* abort_flag = &sm->abort;
  const int h = blockIdx.x / n_ct, ct = blockIdx.x % n_ct;
  const int b0 = blockIdx.y * BN;
  const int nb = min(BN, a.B - b0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tcols = BN <= 32 ? 32 : (BN <= 64 ? 64 : 128);
  const uint32_t a_bytes = 2u * a.d_h * 128, b_bytes = static_cast<uint32_t>(nkb * BN * 128);

  if (threadIdx.x == 0) {
    mbar_init(&sm->full, 1);
    mbar_init(&sm->mma_done, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm->tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem;
  bool mma_issued = false;   // thread 0
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&a.wk_map);
    tma_prefetch_desc(&a.q_map);
    mbar_arrive_expect_tx(&sm->full, a_bytes + b_bytes);
    for (int j = 0; j < 2; ++j)
      tma_load_2d(&a.wk_map, &sm->full, sA + j * a.d_h * 128, ct * kAbsorbM + j * 64, h * a.d_h, l2_evict_first());
  }
  griddep_wait();   // the queries come from the kernel before this one
  const int dq = a.d_h + a.d_rope;
  if (threadIdx.x == 0) {
    for (int kb = 0; kb < nkb; ++kb)
      tma_load_2d(&a.q_map, &sm->full, sB + kb * BN * 128, h * dq + kb * 64, b0, l2_evict_last());
  }
  // with hard / quantised gates each sequence stores its heads by slot (heads
  // whose gate is 0 last, their rows zero); otherwise slot = head
  if (threadIdx.x < nb) {
    int slot = h;
    float on = 1.f;
    const int b = b0 + threadIdx.x;
    if (a.gate_hard) {
      const float* z = a.gate_logits + static_cast<int64_t>(b) * a.H;
      int na = 0;
      slot = head_slot(z, a.H, h, a.gate_mode, a.gate_topk, &na);
      const float gv = head_gate(z, a.H, h, a.gate_mode, a.gate_topk);
      on = gv != 0.f ? 1.f : 0.f;
      if (ct == 0) {
        a.gvals[static_cast<int64_t>(b) * a.H + h] = gv;
        a.head_of_slot[static_cast<int64_t>(b) * a.H + slot] = h;
      }
    }
    sm->slot[threadIdx.x] = slot;
    sm->on[threadIdx.x] = on;
  }
  if (threadIdx.x == 0) {
    if (mbar_wait(&sm->full, 0, abort_flag, a.status)) {
      tc_fence_after();
      // A (MN-major): the two 64-column boxes are d_h * 128 bytes apart; a K step
      // of 16 rows advances 2 KB. B (K-major): box kb holds d_h columns
      // [64 kb, 64 kb + 64); a K step of 16 inside a box advances 32 bytes.
      const uint32_t idesc = idesc_bf16_f32(128, BN, true, false);
      const uint64_t dA = sdesc_sw128(smem_u32(sA), a.d_h * 128, 1024);
      const uint64_t dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      for (int k = 0; k < a.d_h / 16; ++k)
        umma_bf16(tmem, dA + (k * 2048) / 16, dB + ((k >> 2) * BN * 128 + (k & 3) * 32) / 16, idesc, k != 0);
      umma_commit(&sm->mma_done);
      mma_issued = true;
    } else {
      mbar_drain(&sm->full, 0);   // copies still in flight land before the block leaves
    }
  }
  __syncthreads();
  // epilogue: warp w holds latent columns ct*128 + 32 w + lane, one TMEM column per sequence
  bool ok = !*abort_flag && mbar_wait(&sm->mma_done, 0, abort_flag, a.status);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const int row = a.d_c + a.d_rope;
    const int c = ct * kAbsorbM + 32 * warp + lane;
    __nv_bfloat16* qa = static_cast<__nv_bfloat16*>(a.qa);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    for (int n0 = 0; n0 < BN; n0 += 16) {
      uint32_t v[16];
      tmem_ld16(taddr + n0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        if (n < nb)
          qa[(static_cast<int64_t>(b0 + n) * a.H + sm->slot[n]) * row + c] =
              __float2bfloat16_rn(__uint_as_float(v[j]) * a.q_scale * sm->on[n]);
      }
    }
    // decoupled RoPE query dims: copied (already rotated), scaled
    if (ct == 0) {
      const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
      for (int i = threadIdx.x; i < nb * a.d_rope; i += blockDim.x) {
        const int n = i / a.d_rope, r = i % a.d_rope;
        const int64_t src = (static_cast<int64_t>(b0 + n) * a.H + h) * dq + a.d_h + r;
        qa[(static_cast<int64_t>(b0 + n) * a.H + sm->slot[n]) * row + a.d_c + r] =
            __float2bfloat16_rn(__bfloat162float(q[src]) * a.q_scale * sm->on[n]);
      }
    }
  } else if (mma_issued) {
    mbar_drain(&sm->mma_done, 0);   // an issued product completes before TMEM is freed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ---------------------------------------------------------------------------
// 3. attention over the latent cache
// ---------------------------------------------------------------------------
struct DecSmem {
  uint64_t full[6], empty[6];   // per box pair of the ring
  uint64_t rope_full, rope_empty;
  uint64_t q_full, q_empty;
  uint64_t s_full, p_full, o_done, o_free, drain;
  uint64_t never;               // completed by nothing (the stall test hook waits on it)
  uint32_t tmem;
  int abort;
  int vote[3];
  int red[2][4][64];
  float lred[4][64];
  float mfin[64];
};

template <int HG, int NBOX>
struct DecCfg {
  static constexpr bool kRope = NBOX > kNcBox;
  static constexpr int kSG = HG >= 32 ? 2 : 1;              // softmax warp groups (head slices)
  static constexpr int kThreads = 64 + 128 * kSG;
  static constexpr int kQBytes = NBOX * HG * 128;          // absorbed queries, NBOX boxes of [HG x 64]
  static constexpr int kPBytes = kRope ? 0 : HG * 256;     // P [128 tokens x HG]; in the RoPE slot otherwise
  // P is the MN-major B operand of O^T = C^T P^T: token rows of HG bf16 in
  // swizzle atoms of 8 rows (HG 64: 128-byte rows, HG 32: 64, HG 16: 32)
  static constexpr uint32_t kPLayout = HG == 64 ? 2u : (HG == 32 ? 4u : 6u);
  static constexpr int kRopeBytes = kRope ? kBoxBytes : 0;
  static constexpr int kSmemStruct = (static_cast<int>(sizeof(DecSmem)) + 127) & ~127;
  static constexpr int kFixed = kQBytes + kPBytes + kRopeBytes + kSmemStruct + 1024 /*align*/;
  static constexpr int kBudget = 232448;
  static constexpr int kRingMax = (kBudget - kFixed) / kBoxBytes;
  static constexpr int kRing = (kRingMax > 12 ? 12 : kRingMax) & ~1;   // even: box pairs never wrap
  static constexpr int kSmem = kRing * kBoxBytes + kFixed;
  // two S^T buffers of HG columns, then O^T: kNcBox/2 chunks of HG columns
  static constexpr int kTmemCols = (6 * HG <= 128) ? 128 : ((6 * HG <= 256) ? 256 : 512);
  static_assert(kRing >= kNcBox, "ring must hold one tile");
};

// Heads of head group hg that sequence b attends with: all of the group's heads,
// or with hard / quantised gates those whose slot is below the sequence's count
// of active heads (0: the segment is skipped by every role of the block).
__device__ __forceinline__ int seg_heads(const DecodeArgs& a, int b, int hg, int heads_valid) {
  if (!a.gate_hard) return heads_valid;
  const int n = a.n_act[b] - hg * a.HG;
  return n <= 0 ? 0 : (n < heads_valid ? n : heads_valid);
}

template <int HG, int NBOX>
__global__ void __launch_bounds__(64 + 128 * (HG >= 32 ? 2 : 1), 1) decode_attn_kernel(const __grid_constant__ DecodeArgs a) {
  using C = DecCfg<HG, NBOX>;
  constexpr int NR = C::kRing;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* rope_slot = ring + NR * kBoxBytes;
  uint8_t* qs = rope_slot + C::kRopeBytes;
  uint8_t* pbuf = C::kRope ? rope_slot : (qs + C::kQBytes);
  DecSmem* sm = reinterpret_cast<DecSmem*>(qs + C::kQBytes + C::kPBytes);
  volatile int* abort_flag = &sm->abort;

  const int g = blockIdx.x, hg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int heads_valid = min(HG, a.H - hg * HG);

  constexpr int NP = NR / 2;   // ring slots hold box pairs: one full and one empty barrier each
  if (threadIdx.x == 0) {
    for (int i = 0; i < NP; ++i) {
      mbar_init(&sm->full[i], 1);
      mbar_init(&sm->empty[i], 1);
    }
    mbar_init(&sm->rope_full, 1);
    mbar_init(&sm->rope_empty, 1);
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
  const int seg_hi = (seg_lo < a.cta_first_seg[g + 1]) ? a.cta_first_seg[g + 1] : seg_lo;   // empty: no work
  const uint32_t tmem = sm->tmem;
  // S^T of tile n in columns [(n & 1) HG, +HG); O^T from column 2 HG in kNcBox/2 chunks of HG
  const uint32_t tO = tmem + 2 * HG;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    // The whole warp walks the loop: lane 0 waits for free slots and arms the
    // barriers; with a paged cache lane r reads the page of chunk r of the
    // tile (one coalesced read per tile) and issues that chunk's copy.
    if (lane == 0) {
      tma_prefetch_desc(&a.cache_map);
      tma_prefetch_desc(&a.qa_map);
    }
    const uint64_t pol_c = a.n_hg > 1 ? l2_evict_normal() : l2_evict_first();
    const uint64_t pol_q = l2_evict_last();
    const bool paged = a.cache.paged != 0;
    const int ps = paged ? a.cache.page_size : kTileTok;
    uint32_t npair = 0, nrope = 0, nq = 0;
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
          for (int j = 0; j < NBOX; ++j)
            tma_load_2d(&a.qa_map, &sm->q_full, qs + j * HG * 128, j * 64, b * a.H + hg * HG, pol_q);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++nq;
      for (int t = sg.y; t < sg.z && ok; ++t) {
        const int tok0 = t * kTileTok;
        const int valid = min(kTileTok, L - tok0);
        if (C::kRing == kNcBox && !paged && t + 1 < sg.z) {
          // A ring of one tile: each tile's boxes are requested only as the previous
          // weighted sum frees their slots, so the next tile's rows (contiguous in
          // the cache) are brought into L2 now, in NBOX pieces, one per lane.
          const int rows_next = min(kTileTok, L - tok0 - kTileTok);
          const uint32_t row_bytes = static_cast<uint32_t>(a.cache.row) * 2;
          const uint32_t total = static_cast<uint32_t>(rows_next) * row_bytes;   // a multiple of 16
          const uint32_t piece = ((total + NBOX - 1) / NBOX + 15) & ~15u;
          const uint32_t off = static_cast<uint32_t>(lane) * piece;
          if (lane < NBOX && off < total)
            bulk_prefetch_l2(static_cast<const uint8_t*>(a.cache.data) +
                                 (static_cast<int64_t>(b) * a.cache.capacity + tok0 + kTileTok) * row_bytes + off,
                             min(piece, total - off));
        }
        const int nchunk = ps >= kTileTok ? 1 : (valid + ps - 1) / ps;   // <= 16 (page size >= 8)
        int page = 0;
        if (paged && lane < nchunk)
          page = a.cache.block_table[static_cast<int64_t>(b) * a.cache.max_pages_per_seq + (tok0 + lane * ps) / ps];
        const uint32_t tx = ps >= kTileTok ? kBoxBytes : nchunk * ps * 128;
        for (int j = 0; j < NBOX; ++j) {
          // ring boxes go in pairs (one barrier for both); the RoPE box has its own slot
          const bool ring_box = j < kNcBox;
          const uint32_t pslot = npair % NP;
          uint64_t* bar = ring_box ? &sm->full[pslot] : &sm->rope_full;
          uint8_t* dst = ring_box ? ring + (pslot * 2 + (j & 1)) * kBoxBytes : rope_slot;
          if (lane == 0) {
            if (!ring_box) {
              if (nrope > 0 && !mbar_wait(&sm->rope_empty, (nrope - 1) & 1, abort_flag, a.status)) ok = false;
              if (ok) mbar_arrive_expect_tx(bar, tx);
            } else if ((j & 1) == 0) {
              if (npair >= static_cast<uint32_t>(NP) &&
                  !mbar_wait(&sm->empty[pslot], ((npair / NP) & 1) ^ 1, abort_flag, a.status))
                ok = false;
              if (ok) mbar_arrive_expect_tx(bar, 2 * tx);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (!ring_box) ++nrope; else if (j & 1) ++npair;
          if (!paged) {
            if (lane == 0) tma_load_2d(&a.cache_map, bar, dst, j * 64, b * a.cache.capacity + tok0, pol_c);
          } else if (ps >= kTileTok) {
            if (lane == 0) tma_load_3d(&a.cache_map, bar, dst, j * 64, tok0 % ps, page, pol_c);
          } else if (lane < nchunk) {
            tma_load_3d(&a.cache_map, bar, dst + lane * ps * 128, j * 64, 0, page, pol_c);
          }
        }
      }
    }
    if (lane == 0 && *abort_flag) {   // let issued copies land before the block exits
      for (uint32_t c = npair > static_cast<uint32_t>(NP) ? npair - NP : 0; c < npair; ++c)
        mbar_drain(&sm->full[c % NP], (c / NP) & 1);
      if (nrope) mbar_drain(&sm->rope_full, (nrope - 1) & 1);
      if (nq) mbar_drain(&sm->q_full, (nq - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // Per tile: the score MMAs (S^T = C Q^T) of the pairs not yet issued, then
    // while the softmax works on this tile, the first pairs of the next tile
    // (into the other S^T buffer) if their boxes have landed, then the weighted
    // sum O^T += C^T P^T once P is ready, which frees the tile's pairs.
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, HG, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, HG, true, true);
      const uint32_t ring_a = smem_u32(ring), rope_a = smem_u32(rope_slot), q_a = smem_u32(qs),
                     p_a = smem_u32(pbuf);
      uint32_t npair = 0, nrope = 0, ntile = 0, nseg = 0;
      int early = 0;   // pairs of this tile whose score MMAs were issued during the previous tile
      bool ok = true;
      if (a.test_stall && g == 0 && hg == 0) {
        // Test hook: the first CTA's MMA thread waits on a barrier that nothing
        // completes, as it would behind a stalled copy. The bounded wait runs out,
        // raises the block's abort flag and reports a timeout in the status word;
        // every role then leaves through its abort path (copies drained, TMEM freed).
        ok = mbar_wait(&sm->never, 0, abort_flag, a.status);
      }
      // Descriptors are built once; an operand's descriptor is the base one plus its
      // byte offset / 16 (the start-address field cannot carry: shared addresses < 256 KB).
      const uint64_t dRing = sdesc_sw128(ring_a, 16, 1024), dQ = sdesc_sw128(q_a, 16, 1024);
      const uint64_t dRingMN = sdesc_sw128(ring_a, kBoxBytes, 1024);
      const uint64_t dP = sdesc_swz(p_a, kTileTok * HG * 2, 8 * HG * 2, C::kPLayout);   // one atom wide (N = HG)
      auto s_pair = [&](uint32_t c, int p, uint32_t tSb) {   // ring pair c holds boxes 2p, 2p+1
        const uint64_t da = dRing + (c % NP) * (2 * kBoxBytes / 16);
        const uint64_t db = dQ + p * (2 * HG * 128 / 16);
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tSb, da + (b2 * kBoxBytes + kk * 32) / 16, db + (b2 * HG * 128 + kk * 32) / 16, idS,
                      (p | b2 | kk) != 0);
        }
      };
      for (int si = seg_lo; si < seg_hi && ok; ++si) {
        const int4 sg = a.seg_info[si];
        if (seg_heads(a, sg.x, hg, heads_valid) == 0) continue;
        if (!mbar_wait(&sm->q_full, nseg & 1, abort_flag, a.status)) { ok = false; break; }
        for (int t = sg.y; t < sg.z; ++t, ++ntile) {
          const uint32_t tSb = tmem + (ntile & 1) * HG;
          for (int p = early; p < kNcBox / 2; ++p) {
            const uint32_t c = npair + p;
            if (!mbar_wait(&sm->full[c % NP], (c / NP) & 1, abort_flag, a.status)) { ok = false; break; }
            s_pair(c, p, tSb);   // boxes are ordered by their TMA barrier: no tcgen05 fence needed
          }
          if (!ok) break;
          if (C::kRope) {
            if (!mbar_wait(&sm->rope_full, nrope & 1, abort_flag, a.status)) { ok = false; break; }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tSb, sdesc_sw128(rope_a + kk * 32, 16, 1024), dQ + (kNcBox * HG * 128 + kk * 32) / 16, idS,
                        1u);
          }
          if (t + 1 == sg.z) umma_commit(&sm->q_empty);
          umma_commit(&sm->s_full);
          // the next tile of this segment: its first pairs, if they have landed (a
          // non-blocking probe, so a late pair never holds up this tile's weighted sum)
          early = 0;
          if (t + 1 < sg.z) {
            const uint32_t tSn = tmem + ((ntile + 1) & 1) * HG;
            for (int p = 0; p < 2; ++p) {
              const uint32_t c = npair + kNcBox / 2 + p;
              if (!mbar_test(&sm->full[c % NP], (c / NP) & 1)) break;
              s_pair(c, p, tSn);
              ++early;
            }
          }
          // wait for P, then O^T += C^T P^T
          if (!mbar_wait(&sm->p_full, ntile & 1, abort_flag, a.status)) { ok = false; break; }
          const bool first = (t == sg.y);
          if (first && nseg > 0 && !mbar_wait(&sm->o_free, (nseg - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int mc = 0; mc < kNcBox / 2; ++mc) {
            const uint32_t pslot = (npair + mc) % NP;
            const uint64_t da = dRingMN + pslot * (2 * kBoxBytes / 16);
#pragma unroll
            for (int kk = 0; kk < kTileTok / 16; ++kk)
              umma_bf16(tO + mc * HG, da + kk * (2048 / 16), dP + kk * (16 * HG * 2 / 16), idO,
                        (!first || kk > 0) ? 1u : 0u);
            umma_commit(&sm->empty[pslot]);
          }
          if (C::kRope) umma_commit(&sm->rope_empty);
          npair += kNcBox / 2;
          if (C::kRope) ++nrope;
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
    // 4 * SG warps: warp w reads TMEM lane quarter w % 4 (one token row per
    // thread) and owns heads [h0, h0 + HT) of the head group.
    constexpr int SG = C::kSG, HT = HG / SG;
    const int q4 = warp & 3;
    const int h0 = SG == 1 ? 0 : ((warp - 2) >> 2) * HT;
    const int row = q4 * 32 + lane;                      // token row of the tile / latent row of a chunk
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int ltid = threadIdx.x - 64;                   // 0 .. 128 SG - 1
    const float NEG_INF = -__int_as_float(0x7f800000);
    // The softmax warps meet at named barrier 1. After a failed wait a warp
    // keeps walking the same loops (skipping the waits) so every warp executes
    // the same sequence of barriers and the block can exit.
    uint32_t nbox = 0, ntile = 0, nseg = 0;
    bool ok = true;
    for (int si = seg_lo; si < seg_hi; ++si) {
      const int4 sg = a.seg_info[si];
      const int L = sg.w;
      const int S0 = a.seq_starts ? a.seq_starts[sg.x] : 0;
      const int hv = seg_heads(a, sg.x, hg, heads_valid);
      if (hv == 0) continue;
      float m[HT], lsum[HT];
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        m[h] = NEG_INF;
        lsum[h] = 0.f;
      }
      for (int t = sg.y; t < sg.z; ++t, ++ntile) {
        const bool first = (t == sg.y);
        ok = ok && mbar_wait(&sm->s_full, ntile & 1, abort_flag, a.status);
        tc_fence_after();
        // Scores are read from TMEM 16 heads at a time, once for the max test and
        // again for P, so no thread holds all its heads' scores at once.
        const uint32_t tS = tmem + (ntile & 1) * HG + lane_off + h0;
        const int valid = min(kTileTok, L - t * kTileTok);
        // rows of the tile outside [start, L): past the end, or (a context-parallel
        // shard) before the first position this call attends to
        const bool rv = row < valid && t * kTileTok + row >= S0;
        auto load16 = [&](int c, float (&x)[16]) {
          uint32_t v[16];
          tmem_ld16(tS + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) x[j] = rv ? __uint_as_float(v[j]) : NEG_INF;
        };
        bool need = first;
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          float x[16];
          load16(c, x);
#pragma unroll
          for (int j = 0; j < 16; ++j) need |= x[j] > m[c + j] + 8.f;
        }
        // block-wide vote among the softmax threads, one of three slots per tile:
        // after tile n's barrier the slot of tile n - 1 (= n + 2 mod 3) is cleared;
        // its readers finished before this barrier and its next writers (tile n + 2)
        // come after the barrier of tile n + 1, so no vote can be erased
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
            if (rescale) {
              // O^T columns of these heads scale by alpha (O of the previous tile is
              // complete: S of this tile was committed after it)
#pragma unroll 1
              for (int mc = 0; mc < kNcBox / 2; ++mc) {
                uint32_t v[16];
                tmem_ld16(tO + lane_off + mc * HG + h0 + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha[j]);
                tmem_st16(tO + lane_off + mc * HG + h0 + c, v);
              }
              tmem_st_wait();
            }
          }
        }
        // P = exp2(s - m) as bf16, this thread's token row of P[token][head]: 16-byte
        // chunks of 8 heads, chunk index XOR the row bits of the swizzle atom
        uint8_t* pb = pbuf + row * (HG * 2);
        const int sw = HG == 64 ? (row & 7) : (HG == 32 ? ((row >> 1) & 3) : ((row >> 2) & 1));
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          float x[16];
          load16(c, x);
#pragma unroll
          for (int c8 = 0; c8 < 16; c8 += 8) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const int h = c + c8 + k;
              const float p0 = rv ? ex2_approx(x[c8 + k] - m[h]) : 0.f;
              const float p1 = rv ? ex2_approx(x[c8 + k + 1] - m[h + 1]) : 0.f;
              lsum[h] += p0;
              lsum[h + 1] += p1;
              w[k >> 1] = pack_bf16x2(p0, p1);
            }
            const int chunk = ((h0 + c + c8) >> 3) ^ sw;
            *reinterpret_cast<uint4*>(pb + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (!rv) {
          // rows past the sequence end may hold anything: zero them so 0 * garbage cannot reach O
#pragma unroll 1
          for (int j = h0 / HT; j < kNcBox; j += SG) {
            uint8_t* box = ring + ((nbox + j) % NR) * kBoxBytes + row * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) reinterpret_cast<uint4*>(box)[c] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm->p_full);
        nbox += kNcBox;
      }
      // ---- segment end: write the partial (unnormalised O, running max m, sum l)
      ok = ok && mbar_wait(&sm->o_done, nseg & 1, abort_flag, a.status);
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        float v = lsum[h];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) sm->lred[q4][h0 + h] = v;
        if (SG > 1 && lane == 0 && q4 == 0) sm->mfin[h0 + h] = m[h];   // the running max is the same in every row
      }
      asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");
      const int64_t pbase = (static_cast<int64_t>(hg) * a.max_seg + si) * HG;
      if (ok && ltid < hv) {
        float l = 0.f, mh = NEG_INF;
        if (SG == 1) {   // every thread holds the running max of every head
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
      for (int mc = 0; mc < kNcBox / 2; ++mc) {
#pragma unroll
        for (int c = 0; c < HT; c += 16) {
          uint32_t v[16];
          tmem_ld16(tO + lane_off + mc * HG + h0 + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (ok && h0 + c + j < hv)
              a.o_part[(pbase + h0 + c + j) * kDc + mc * 128 + row] = __uint_as_float(v[j]);
          }
        }
      }
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"n"(128 * SG) : "memory");   // lred / mfin reuse
      mbar_arrive(&sm->o_free);
      ++nseg;
    }
  }

  // one lane of a warp ran a role alone: reconverge before the block-wide barrier
  // (a partly arrived warp must not count as arrived)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// 4. merge the split-K partials of each (head, sequence) by their log-sum-exp
//    weights: O_lat = sum_i 2^(m_i - m) O_i / sum_i 2^(m_i - m) l_i, written as
//    bf16 [H, B, d_c] for the W_v product (a tensor-core GEMM with the gate in
//    its epilogue). Block (0, 0) also clears that GEMM's split-K tickets.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_merge_kernel(DecodeArgs a) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int slot = blockIdx.x, b = blockIdx.y;
  const int hg = slot / a.HG, hl = slot % a.HG;
  if (slot == 0 && b == 0)
    for (int i = threadIdx.x; i < a.n_gemm_tiles; i += blockDim.x) a.gemm_counters[i] = 0;
  int h = slot;
  if (a.gate_hard) {
    // slot -> head; a head whose gate is 0 was skipped: its latent output is 0
    h = a.head_of_slot[static_cast<int64_t>(b) * a.H + slot];
    if (slot >= a.n_act[b]) {
      if (a.partial_out) {   // an empty partial: O = 0, log-sum-exp -inf
        float* dst = a.partial_out + (static_cast<int64_t>(b) * a.H + h) * (kDc + kPartialPad);
        for (int j = threadIdx.x; j < kDc + kPartialPad; j += blockDim.x)
          dst[j] = j == kDc ? -__int_as_float(0x7f800000) : 0.f;
        return;
      }
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.olat) + (static_cast<int64_t>(h) * a.B + b) * kDc;
      for (int j = threadIdx.x; j < kDc; j += blockDim.x) dst[j] = __float2bfloat16_rn(0.f);
      return;
    }
  }
  const int s0 = a.seq_first_seg[b], s1 = a.seq_first_seg[b + 1];
  const int64_t base = static_cast<int64_t>(hg) * a.max_seg;
  // one pass over the segments, rescaling the running sums when the max grows
  // (every iteration's loads are independent of the previous ones)
  float mx = -__int_as_float(0x7f800000), l = 0.f;
  float acc[kDc / 128];
#pragma unroll
  for (int j = 0; j < kDc / 128; ++j) acc[j] = 0.f;
  for (int s = s0; s < s1; ++s) {
    const float* ml = a.ml_part + ((base + s) * a.HG + hl) * 2;
    const float* op = a.o_part + ((base + s) * a.HG + hl) * kDc;
    const float ms = ml[0], ls = ml[1];
    float o[kDc / 128];
#pragma unroll
    for (int j = 0; j < kDc / 128; ++j) o[j] = __ldcg(op + j * 128 + threadIdx.x);
    const float mn = fmaxf(mx, ms);
    const float a_old = (mx == -__int_as_float(0x7f800000)) ? 0.f : ex2_approx(mx - mn);
    const float a_new = (ms == -__int_as_float(0x7f800000)) ? 0.f : ex2_approx(ms - mn);
    l = l * a_old + ls * a_new;
#pragma unroll
    for (int j = 0; j < kDc / 128; ++j) acc[j] = acc[j] * a_old + o[j] * a_new;
    mx = mn;
  }
  const float inv = (s1 > s0 && l > 0.f) ? 1.f / l : 0.f;
  if (a.partial_out) {
    // context-parallel share: normalised O_lat of this share and its log-sum-exp
    // (log2 domain), merged across shares by decode_merge_ranks
    float* dst = a.partial_out + (static_cast<int64_t>(b) * a.H + h) * (kDc + kPartialPad);
#pragma unroll
    for (int j = 0; j < kDc / 128; ++j) dst[j * 128 + threadIdx.x] = acc[j] * inv;
    if (threadIdx.x < kPartialPad)
      dst[kDc + threadIdx.x] = threadIdx.x == 0 ? ((l > 0.f) ? mx + __log2f(l) : -__int_as_float(0x7f800000)) : 0.f;
    return;
  }
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.olat) + (static_cast<int64_t>(h) * a.B + b) * kDc;
#pragma unroll
  for (int j = 0; j < kDc / 128; ++j) dst[j * 128 + threadIdx.x] = __float2bfloat16_rn(acc[j] * inv);
}

// ---------------------------------------------------------------------------
// 5. context-parallel merge: the shares of one sequence's cache held by R
//    ranks each give (O_r normalised, lse_r); O = sum_r 2^(lse_r - M) O_r /
//    sum_r 2^(lse_r - M), M = max_r lse_r. One block per (head, sequence).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_merge_ranks_kernel(MergeRanksArgs a) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int h = blockIdx.x, b = blockIdx.y;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const int64_t row = static_cast<int64_t>(b) * a.H + h;
  const int64_t rank_stride = static_cast<int64_t>(a.B) * a.H * (kDc + kPartialPad);
  float mx = NEG_INF, wsum = 0.f;
  float acc[kDc / 128];
#pragma unroll
  for (int j = 0; j < kDc / 128; ++j) acc[j] = 0.f;
  for (int r = 0; r < a.R; ++r) {
    const float* src = a.partials + r * rank_stride + row * (kDc + kPartialPad);
    const float lse = __ldcg(src + kDc);
    if (lse == NEG_INF) continue;   // an empty share
    float o[kDc / 128];
#pragma unroll
    for (int j = 0; j < kDc / 128; ++j) o[j] = __ldcg(src + j * 128 + threadIdx.x);
    const float mn = fmaxf(mx, lse);
    const float a_old = (mx == NEG_INF) ? 0.f : ex2_approx(mx - mn);
    const float a_new = ex2_approx(lse - mn);
    wsum = wsum * a_old + a_new;
#pragma unroll
    for (int j = 0; j < kDc / 128; ++j) acc[j] = acc[j] * a_old + o[j] * a_new;
    mx = mn;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.olat) + (static_cast<int64_t>(h) * a.B + b) * kDc;
#pragma unroll
  for (int j = 0; j < kDc / 128; ++j) dst[j * 128 + threadIdx.x] = __float2bfloat16_rn(acc[j] * inv);
  if (a.gate_hard && threadIdx.x == 0)
    a.gvals[row] = head_gate(a.gate_logits + static_cast<int64_t>(b) * a.H, a.H, h, a.gate_mode, a.gate_topk);
}

cudaError_t launch_decode_merge_ranks(const MergeRanksArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  prof_begin(st, "decode_merge_ranks");
  cudaError_t e = launch_pdl(decode_merge_ranks_kernel, dim3(a.H, a.B), dim3(128), 0, st, 1, a);
  prof_end(st);
  return e;
}

}  // namespace gmla

#include "decode_fp8.cuh"

namespace gmla {

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

DecodeLayout decode_layout(int B, int H, int eff_heads, int d_h, int d_c, int d_rope, int num_sms, bool fp8) {
  DecodeLayout L{};
  const int E = eff_heads;
  L.HG = E <= 16 ? 16 : (E % 64 == 0 ? 64 : (E % 32 == 0 ? 32 : 16));
  if (fp8 && L.HG > 32) L.HG = 32;   // hi and lo columns of 64 heads would not fit tensor memory
  L.n_hg = (E + L.HG - 1) / L.HG;
  // the FP8 kernel with 16 heads runs two CTAs per SM
  L.G = ((fp8 && L.HG == 16) ? 2 : 1) * num_sms / L.n_hg;
  if (L.G < 1) L.G = 1;
  L.max_seg = L.G + B + 1;
  const size_t row = static_cast<size_t>(d_c + d_rope);
  size_t off = 256;   // status word
  L.off_qa = off;
  {
    const size_t bf16_q = static_cast<size_t>(B) * H * row * 2 + 16 * row * 2;   // + padded head rows
    const size_t fp8_q = static_cast<size_t>(B) * ((H + L.HG - 1) / L.HG) * 2 * L.HG * d_c;
    off = align256(off + (fp8 ? (fp8_q > bf16_q ? fp8_q : bf16_q) : bf16_q));
  }
  L.off_opart = off;
  off = align256(off + static_cast<size_t>(L.n_hg) * L.max_seg * L.HG * kDc * 4);
  L.off_ml = off;
  off = align256(off + static_cast<size_t>(L.n_hg) * L.max_seg * L.HG * 2 * 4);
  L.off_seg = off;
  off = align256(off + static_cast<size_t>(L.max_seg) * sizeof(int4));
  L.off_seqfirst = off;
  off = align256(off + static_cast<size_t>(B + 1) * 4);
  L.off_ctafirst = off;
  off = align256(off + static_cast<size_t>(L.G + 1) * 4);
  L.off_olat = off;
  off = align256(off + static_cast<size_t>(H) * B * d_c * 2);
  L.off_gemm = off;
  L.gemm_plan = gemm_swap_plan(H * d_h / 128, B, d_c, num_sms);
  off = align256(off + L.gemm_plan.ws_bytes);
  L.off_gvals = off;
  off = align256(off + static_cast<size_t>(B) * H * 4);
  L.off_hslot = off;
  off = align256(off + static_cast<size_t>(B) * H * 4);
  L.off_nact = off;
  off = align256(off + static_cast<size_t>(B) * 4);
  L.off_qmul = off;
  off = align256(off + static_cast<size_t>(B) * H * 4);
  L.total = off;
  return L;
}

template <int HG, int NBOX>
static cudaError_t launch_attn(const DecodeArgs& a, cudaStream_t st) {
  using C = DecCfg<HG, NBOX>;
  auto k = decode_attn_kernel<HG, NBOX>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  prof_begin(st, "decode_attn");
  e = launch_pdl(k, dim3(a.G, a.n_hg), dim3(C::kThreads), C::kSmem, st, 1, a);
  prof_end(st);
  return e;
}

static cudaError_t launch_decode_fp8(DecodeArgs& a, cudaStream_t st) {
  const int n_absorb = a.H * ((a.B + kAbs8B - 1) / kAbs8B);
  prof_begin(st, "decode_absorb_plan");
  cudaError_t e = launch_pdl(decode_absorb_fp8_kernel, dim3(n_absorb + 1), dim3(256), 0, st, 1, a);
  prof_end(st);
  if (e != cudaSuccess) return e;
  switch (a.HG) {
    case 16: e = launch_attn_fp8<16>(a, st); break;
    case 32: e = launch_attn_fp8<32>(a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  prof_begin(st, "decode_merge");
  e = launch_pdl(decode_merge_kernel, dim3(a.H, a.B), dim3(128), 0, st, 1, a);
  prof_end(st);
  return e;
}

int absorb_tile_n(int B) { return B >= 128 ? 128 : ((B + 15) / 16) * 16; }

cudaError_t launch_decode_bf16(DecodeArgs& a, cudaStream_t st) {
  if (a.fp8) return launch_decode_fp8(a, st);
  const size_t smem = absorb_smem_bytes(a.d_h, a.absorb_bn);
  cudaError_t e = cudaFuncSetAttribute(decode_absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  prof_begin(st, "decode_absorb_plan");
  e = launch_pdl(decode_absorb_tc_kernel, dim3(a.H * (a.d_c / kAbsorbM) + 1, (a.B + a.absorb_bn - 1) / a.absorb_bn),
                 dim3(128), smem, st, 1, a);
  prof_end(st);
  if (e != cudaSuccess) return e;
  const int nbox = (a.d_c + a.d_rope) / 64;
  switch (a.HG * 16 + nbox) {
    case 16 * 16 + 8: e = launch_attn<16, 8>(a, st); break;
    case 16 * 16 + 9: e = launch_attn<16, 9>(a, st); break;
    case 32 * 16 + 8: e = launch_attn<32, 8>(a, st); break;
    case 32 * 16 + 9: e = launch_attn<32, 9>(a, st); break;
    case 64 * 16 + 8: e = launch_attn<64, 8>(a, st); break;
    case 64 * 16 + 9: e = launch_attn<64, 9>(a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  prof_begin(st, "decode_merge");
  e = launch_pdl(decode_merge_kernel, dim3(a.H, a.B), dim3(128), 0, st, 1, a);
  prof_end(st);
  return e;
}

}  // namespace gmla
