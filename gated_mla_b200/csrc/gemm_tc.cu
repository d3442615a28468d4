// gemm_tc.cu — bf16 GEMM on tcgen05 tensor cores with fused epilogues.
//
// D = X W^T for an activation X [T, K] and a weight that is a list of up to
// kMaxSeg segments W_s [rows_s, K] (all K-major, row-major [out, in]). Each
// segment has its own epilogue (plain store, fp32 + bias, RoPE, scatter into
// the latent cache). Used for:
//   * x -> [c | k^R | q | q^R | gate logits]   ("Gated MLA 计算公式" §一/§二;
//                                                "精读笔记 03" §5.2)
//   * latent rows -> K^(h), V^(h) for prefill    ("Gated MLA 计算公式" §一)
//   * gated o -> y = W_o (...)                    ("Gated MLA 计算公式" §二 boxed eq.)
//
// Two orientations share one kernel:
//   kSwap = true  (few tokens): MMA M = 128 weight rows, N = BN tokens.
//   kSwap = false (many tokens): MMA M = 128 token rows, N = BN weight rows.
// Roles: warp 0 issues TMA loads into a ring of shared-memory stages, warp 1
// allocates TMEM and one thread issues the MMAs, warps 2..5 drain the fp32
// accumulator from TMEM and run the epilogue. Every wait is bounded. In the
// many-token orientation two CTAs share an SM, so that one CTA's epilogue runs
// while the other's MMAs keep the tensor pipe busy.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gmla {

template <int BN, bool kSwap>
struct GemmCfg {
  static constexpr int kABytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;               // BN rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  // Few tokens (weight streaming): 4 stages, narrow tiles let two CTAs share an SM.
  // Many tokens: two CTAs per SM with 96 KB of stages each, so one CTA's epilogue
  // runs while the other's MMAs keep the tensor pipe busy.
  static constexpr int kStages = kSwap ? ((BN >= 256) ? 4 : (BN >= 128 ? 6 : 4)) : (BN >= 256 ? 2 : 3);
  static constexpr int kCtasPerSm = kSwap ? 1 : 2;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/ + 12 * BN;
  // split-K partials are received into the (then idle) stage memory:
  // splits x 128 x cpr fp32 with splits <= 8 and cpr = ceil4(ceil(BN / splits)) <= BN / splits + 3
  static_assert(!kSwap || 128 * 4 * (BN + 24) <= kStages * kStageBytes, "split-K receive buffer");
};

struct GemmTile {
  int seg;       // weight segment
  int wrow0;     // first weight row of the tile (segment-local)
  int tok0;      // first token index (packed) of the tile
  int act_row0;  // first activation row read by TMA
  int ntok;      // valid tokens in this tile
};

// Large-token orientation: blocks are taken in groups of kGroupT token tiles,
// the token tile varying fastest, so that the blocks resident at once share
// few weight tiles and few token tiles and both stay in L2 (the plain order
// would stream every weight tile from HBM once per token tile).
constexpr int kGroupT = 16;

template <int BN, bool kSwap>
__device__ __forceinline__ bool gemm_tile(const GemmArgs& a, GemmTile& t) {
  int wt = blockIdx.x, tt = blockIdx.y;
  if (!kSwap) {
    const int nw = gridDim.x, nt = gridDim.y;
    const int lin = blockIdx.y * nw + blockIdx.x;
    const int group = lin / (kGroupT * nw);
    const int first = group * kGroupT;
    const int gsize = min(kGroupT, nt - first);
    const int in = lin - group * kGroupT * nw;
    tt = first + in % gsize;
    wt = in / gsize;
  }
  int s = 0;
  while (s + 1 < a.n_seg && wt >= a.seg_tile_begin[s + 1]) ++s;
  t.seg = s;
  constexpr int kWTile = kSwap ? 128 : BN;
  constexpr int kTTile = kSwap ? BN : 128;
  t.wrow0 = (wt - a.seg_tile_begin[s]) * kWTile;
  if (a.row_mode == 0) {
    t.tok0 = tt * kTTile;
    t.act_row0 = t.tok0;
    t.ntok = min(kTTile, a.T - t.tok0);
  } else if (a.row_mode == 2) {
    t.tok0 = tt * kTTile;
    t.act_row0 = (a.seg_tile_begin[s] * kWTile + t.wrow0) / a.rows_per_group * a.act_group_stride + t.tok0;
    t.ntok = min(kTTile, a.T - t.tok0);
  } else {
    // prefill sequence tiles: token tile -> (sequence, offset)
    const int b = tt / a.tiles_per_seq;
    const int t0 = (tt % a.tiles_per_seq) * kTTile;
    const int beg = a.cu_seqlens[b], len = a.cu_seqlens[b + 1] - beg;
    t.tok0 = beg + t0;
    t.act_row0 = b * a.act_seq_stride + t0;
    t.ntok = min(kTTile, len - t0);
  }
  return t.ntok > 0;
}

template <int BN, bool kSwap>
__global__ void __launch_bounds__(192, kSwap ? 1 : 2) gemm_bf16_tc_kernel(const __grid_constant__ GemmArgs a) {
  using C = GemmCfg<BN, kSwap>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* drain = acc_full + 1;
  uint64_t* red_full = drain + 1;   // split-K: the partials addressed to this CTA have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // per-token output row and position of this tile (swap orientation), filled once
  int64_t* tok_row = reinterpret_cast<int64_t*>(smem + C::kStages * C::kStageBytes + 256);
  int* tok_pos = reinterpret_cast<int*>(tok_row + (kSwap ? BN : 1));

  if (a.row_mode == 1) griddep_wait();   // the tile reads the sequence offsets
  GemmTile tile;
  if (!gemm_tile<BN, kSwap>(a, tile)) return;   // uniform across the block

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {   // start the descriptor fetches while the block sets up
    tma_prefetch_desc(&a.act);
    tma_prefetch_desc(&a.wt[tile.seg]);
  }
  const int num_kb_total = (a.K + 63) / 64;
  const int kbps = (kSwap && a.kb_per_split > 0) ? a.kb_per_split : num_kb_total;
  const int kb_begin = kSwap ? blockIdx.z * kbps : 0;
  const int num_kb = kSwap ? min(num_kb_total - kb_begin, kbps) : num_kb_total;
  // split-K (swap orientation): the K splits of a tile form a cluster along z;
  // rank z owns the accumulator columns [z*cpr, (z+1)*cpr) of the tile
  const bool split = kSwap && a.splits > 1;
  const int cpr = ((BN + a.splits - 1) / a.splits + 3) & ~3;
  const uint32_t rank = split ? cluster_ctarank() : 0u;
  const int own_cols = split ? max(0, min(cpr, BN - static_cast<int>(rank) * cpr)) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(red_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (split) mbar_arrive_expect_tx(red_full, a.splits * 128 * own_cols * 4);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;

  float gl0[16];   // epilogue warps, swap orientation: see below
  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* wmap = &a.wt[tile.seg];
      tma_prefetch_desc(&a.act);
      tma_prefetch_desc(wmap);
      const uint64_t pol_w = l2_evict_normal();
      const uint64_t pol_x = l2_evict_last();
      // Weight tiles are never written by a kernel: those of the first stages
      // are requested before waiting for the kernel that produces the activations.
      const int pre = min(num_kb, C::kStages);
      for (int kb = 0; kb < pre; ++kb) {
        uint8_t* sa = smem + kb * C::kStageBytes;
        mbar_arrive_expect_tx(&full[kb], C::kStageBytes);
        if (kSwap)
          tma_load_2d(wmap, &full[kb], sa, (kb_begin + kb) * 64, tile.wrow0, pol_w);
        else
          tma_load_2d(wmap, &full[kb], sa + C::kABytes, kb * 64, tile.wrow0, pol_w);
      }
      griddep_wait();
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int st = kb % C::kStages;
        if (kb >= C::kStages &&
            !mbar_wait(&empty[st], ((kb / C::kStages) & 1) ^ 1, abort_flag, a.status))
          break;
        uint8_t* sa = smem + st * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        if (kb >= pre) mbar_arrive_expect_tx(&full[st], C::kStageBytes);
        if (kSwap) {
          if (kb >= pre) tma_load_2d(wmap, &full[st], sa, (kb_begin + kb) * 64, tile.wrow0, pol_w);
          tma_load_2d(&a.act, &full[st], sb, (kb_begin + kb) * 64, tile.act_row0, pol_x);
        } else {
          tma_load_2d(&a.act, &full[st], sa, kb * 64, tile.act_row0, pol_x);
          if (kb >= pre) tma_load_2d(wmap, &full[st], sb, kb * 64, tile.wrow0, pol_w);
        }
        ++issued;
      }
      if (issued < pre) issued = pre;   // stages armed and partly loaded before the wait
      if (*abort_flag) {   // let copies still in flight land before the block exits
        for (int kb = max(0, issued - C::kStages); kb < issued; ++kb)
          mbar_drain(&full[kb % C::kStages], (kb / C::kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      bool ok = true;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int st = kb % C::kStages;
        if (!mbar_wait(&full[st], (kb / C::kStages) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        // the stage is ordered by its TMA barrier; a tcgen05 fence per stage would
        // drain the tensor pipe between k-blocks
        const uint32_t sa = smem_u32(smem + st * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          umma_bf16(tmem, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kb | kk) != 0);
        }
        umma_commit(&empty[st]);
      }
      if (ok) {
        umma_commit(acc_full);
      } else {
        umma_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarter (warp % 4)
    const int q = warp & 3;
    const int r = q * 32 + lane;            // accumulator row of this thread
    griddep_wait();                         // before reading positions or writing outputs
    // by value: a runtime-indexed reference into the parameter space costs a
    // chain of constant-bank loads on every use
    const EpiSeg e = a.epi[tile.seg];
    const int seg_rows = a.seg_rows[tile.seg];
    if (kSwap) {
      // While the MMAs run: the tile's token -> output row / position table (built
      // once in shared memory so the store loop has no dependent global loads), and
      // the gate-logit lines this warp will read brought into L1.
      for (int lt = threadIdx.x - 64; lt < BN; lt += 128) {
        const int tok = tile.tok0 + lt;
        int64_t row = tok;
        int pos = 0;
        if (lt < tile.ntok && (e.rope || e.cache_scatter)) pos = a.positions[tok];
        if (lt < tile.ntok && e.cache_scatter) {
          row = cache_row(a.cache, a.seq_ids[tok], pos);
          if (row < 0) report_status(a.status, kStatusRange);
        }
        tok_row[lt] = lt < tile.ntok ? row : -1;
        tok_pos[lt] = pos;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
    }
    // the gate logits of the first 16 tokens this thread stores (all of them in the
    // few-token case), loaded before the accumulator is ready
    {
      const int f = tile.wrow0 + r;
      const int c_lo = split ? static_cast<int>(rank) * cpr : 0;
      const int c_hi = split ? c_lo + own_cols : BN;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int lt = c_lo + j;
        gl0[j] = (kSwap && e.gate && f < seg_rows && lt < c_hi && lt < tile.ntok)
                     ? e.gate[static_cast<int64_t>(tile.tok0 + lt) * e.gate_stride + f / e.gate_div]
                     : 0.f;
      }
    }
    // Split-K epilogues meet at named barrier 2; a failed wait still walks the
    // same barriers (with its stores skipped) so the four warps stay in step.
    // warp-uniform: the TMEM loads below are warp-collective
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, a.status));
    if (acc_ok || kSwap) {
      tc_fence_after();
      if (kSwap) {
        // row r = weight feature, columns = tokens
        const int f = tile.wrow0 + r;
        // this thread's feature is fixed: hoist its column offset, bias and gate index
        const int64_t colpart =
            static_cast<int64_t>(f / e.block) * e.block_stride + (f % e.block) + e.col_offset;
        const bool f_ok = f < seg_rows;
        const float fbias = (e.bias && f_ok) ? e.bias[f] : 0.f;
        const int gcol = e.gate ? f / e.gate_div : 0;
        auto store_chunk = [&](int c0, float (&x)[16]) {
          // the gate logits of the 16 tokens, all requested before any store
          // (the compiler cannot move them past stores that might alias)
          float gl[16];
          if (e.gate) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              gl[j] = c0 == 0 ? gl0[j]
                              : ((tok_row[c0 + j] >= 0 && f_ok)
                                     ? e.gate[static_cast<int64_t>(tile.tok0 + c0 + j) * e.gate_stride + gcol]
                                     : 0.f);
          }
#pragma unroll 4
          for (int j = 0; j < 16; ++j) {
            const int tl = c0 + j;
            float val = x[j];
            if (e.rope) {
              const float partner = __shfl_xor_sync(0xffffffffu, val, 1);
              const int fi = f % e.block;
              val = rope_rotate(val, partner, fi & 1, tok_pos[tl], fi >> 1, e.block, a.log2_rope_base);
            }
            const int64_t row = tok_row[tl];
            if (row < 0 || !f_ok) continue;
            val += fbias;
            if (e.gate) val *= e.gate_value ? gl[j] : __fdividef(1.f, 1.f + __expf(-gl[j]));
            const int64_t off = row * e.row_stride + colpart;
            store_out(e, off, val);
          }
        };
        if (!split) {
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
            tmem_ld_wait();
            float x[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = __uint_as_float(v[j]);
            if (acc_ok) store_chunk(c0, x);
          }
        }
        // (split-K: the accumulator is pushed to the owning CTAs below)
      } else {
        // row r = token, columns = weight features
        const bool tok_ok = r < tile.ntok;
        const int tok = tile.tok0 + r;
        int pos = 0;
        int64_t row = tok;
        if (tok_ok && (e.rope || e.cache_scatter)) pos = a.positions[tok];
        if (tok_ok && e.cache_scatter) {
          row = cache_row(a.cache, a.seq_ids[tok], pos);
          if (row < 0) report_status(a.status, kStatusRange);
        }
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
          tmem_ld_wait();
          if (!tok_ok || row < 0) continue;
          const int f0 = tile.wrow0 + c0;
          float x[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) x[j] = __uint_as_float(v[j]);
          if (e.rope) {
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const int fi = (f0 + j) % e.block;
              const float x0 = x[j], x1 = x[j + 1];
              x[j] = rope_rotate(x0, x1, false, pos, fi >> 1, e.block, a.log2_rope_base);
              x[j + 1] = rope_rotate(x1, x0, true, pos, fi >> 1, e.block, a.log2_rope_base);
            }
          }
          const int64_t off16 = row * e.row_stride + static_cast<int64_t>(f0 / e.block) * e.block_stride +
                                (f0 % e.block) + e.col_offset;
          const bool whole = !e.gate && (f0 + 16 <= seg_rows) && (f0 % e.block) + 16 <= e.block;
          const bool vec = whole && !e.out_f32 && !e.out_fp8 && !e.bias && off16 % 8 == 0;
          const bool vec32 = whole && e.out_f32 && off16 % 4 == 0;   // fp32 rows (+ bias), 16-byte stores
          if (vec32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(e.out) + off16);
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              float4 o = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
              if (e.bias) {
                const float4 bb = __ldg(reinterpret_cast<const float4*>(e.bias + f0 + j));
                o.x += bb.x;
                o.y += bb.y;
                o.z += bb.z;
                o.w += bb.w;
              }
              dst[j >> 2] = o;
            }
          } else if (vec) {
            const int64_t off = off16;
            uint4 p0, p1;
            p0.x = pack_bf16x2(x[0], x[1]);
            p0.y = pack_bf16x2(x[2], x[3]);
            p0.z = pack_bf16x2(x[4], x[5]);
            p0.w = pack_bf16x2(x[6], x[7]);
            p1.x = pack_bf16x2(x[8], x[9]);
            p1.y = pack_bf16x2(x[10], x[11]);
            p1.z = pack_bf16x2(x[12], x[13]);
            p1.w = pack_bf16x2(x[14], x[15]);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(e.out) + off);
            dst[0] = p0;
            dst[1] = p1;
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (f0 + j < seg_rows) epi_store(e, row, f0 + j, x[j], tok);
          }
        }
      }
    }
  }

  if (split) {
    // Every split of the tile has finished its MMAs once the cluster barrier
    // completes, so their stage memory is idle and receives the partials:
    // recv[src split][row][cpr] fp32. Each split pushes the columns that rank
    // z owns straight from its accumulator to rank z (st.async, completing
    // bytes on rank z's red_full); the owner sums the splits and stores.
    // A second cluster barrier, split into an arrive after the sends and a wait
    // before the block exits, keeps every CTA resident until all of its peers
    // have issued what they send to it, also when an owner's wait for its
    // partials gave up. Nothing between the two halves waits without a bound,
    // so the final wait ends once every CTA has issued its sends.
    __syncwarp();   // warps whose role ran on one lane arrive whole at the aligned barrier
    cluster_sync_all();
    float* recv = reinterpret_cast<float*>(smem);
    if (warp >= 2) {
      const int q = warp & 3, r = q * 32 + lane;
      const bool acc_ok = __all_sync(0xffffffffu, !*abort_flag);
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 16; g += 4) {
          const int col = c0 + g;
          const uint32_t z = static_cast<uint32_t>(col / cpr);
          const float4 x = acc_ok ? make_float4(__uint_as_float(v[g]), __uint_as_float(v[g + 1]),
                                                __uint_as_float(v[g + 2]), __uint_as_float(v[g + 3]))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          const uint32_t dst = smem_u32(recv + (rank * 128 + r) * cpr + (col - static_cast<int>(z) * cpr));
          st_async_v4(cluster_map(dst, z), x, cluster_map(smem_u32(red_full), z));
        }
      }
    }
    cluster_arrive_release();   // every thread: this CTA's sends are issued
    if (warp >= 2) {
      const int q = warp & 3, r = q * 32 + lane;
      if (own_cols > 0) {
        const bool got = mbar_wait_cluster(red_full, 0, abort_flag, a.status);
        const int col0 = static_cast<int>(rank) * cpr;
        const int f = tile.wrow0 + r;
        const EpiSeg e = a.epi[tile.seg];
        const int seg_rows = a.seg_rows[tile.seg];
        const bool f_ok = f < seg_rows;
        const int64_t colpart = static_cast<int64_t>(f / e.block) * e.block_stride + (f % e.block) + e.col_offset;
        const float fbias = (e.bias && f_ok) ? e.bias[f] : 0.f;
        const int gcol = e.gate ? f / e.gate_div : 0;
#pragma unroll 1
        for (int c = 0; c < own_cols; c += 16) {
          const int nc = min(16, own_cols - c);   // a multiple of 4
          // gate logits of these tokens, all requested before any store
          float gl[16];
          if (e.gate) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int tl = col0 + c + j;
              gl[j] = c == 0 ? gl0[j]
                             : ((j < nc && tok_row[tl] >= 0 && f_ok)
                                    ? e.gate[static_cast<int64_t>(tile.tok0 + tl) * e.gate_stride + gcol]
                                    : 0.f);
            }
          }
          float x[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) x[j] = 0.f;
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            if (z >= a.splits) break;
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              if (j >= nc) break;
              const float4 u = *reinterpret_cast<const float4*>(recv + (z * 128 + r) * cpr + c + j);
              x[j] += u.x;
              x[j + 1] += u.y;
              x[j + 2] += u.z;
              x[j + 3] += u.w;
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j >= nc) break;
            const int tl = col0 + c + j;
            float val = x[j];
            if (e.rope) {
              const float partner = __shfl_xor_sync(0xffffffffu, val, 1);
              const int fi = f % e.block;
              val = rope_rotate(val, partner, fi & 1, tok_pos[tl], fi >> 1, e.block, a.log2_rope_base);
            }
            const int64_t row = tok_row[tl];
            if (row < 0 || !f_ok || !got) continue;
            val += fbias;
            if (e.gate) val *= e.gate_value ? gl[j] : __fdividef(1.f, 1.f + __expf(-gl[j]));
            const int64_t off = row * e.row_stride + colpart;
            store_out(e, off, val);
          }
        }
      }
    }
    cluster_wait_acquire();   // no CTA leaves while a peer may still send into it
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

template <int BN, bool kSwap>
static cudaError_t launch_one(const GemmArgs& a, dim3 grid, cudaStream_t st, const char* name) {
  using C = GemmCfg<BN, kSwap>;
  auto k = gemm_bf16_tc_kernel<BN, kSwap>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  prof_begin(st, name);
  // the K splits of one tile (swap orientation) run as a cluster along z
  e = launch_pdl(k, grid, dim3(192), C::kSmemBytes, st, (kSwap && a.splits > 1) ? a.splits : 1, a);
  prof_end(st);
  return e;
}

int gemm_weight_tile(bool swap, int bn) { return swap ? 128 : bn; }

int gemm_swap_bn(int T) { return T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : T <= 128 ? 128 : 256; }

SwapPlan gemm_swap_plan(int wtiles, int T, int K, int num_sms) {
  SwapPlan p{};
  p.bn = gemm_swap_bn(T);
  p.ttiles = (T + p.bn - 1) / p.bn;
  const int tiles = wtiles * p.ttiles;
  const int num_kb = (K + 63) / 64;
  // Few tiles: split K (one cluster of splits per tile) until the tiles fill one
  // CTA per SM. Many tiles: split so there are at least four waves of two CTAs
  // per SM (tail imbalance < 25%).
  // With a long K (each split would keep >= 16 K blocks at two CTAs per SM), about
  // 1.5 CTAs per SM: more weight streams in flight than one per SM, while every
  // CTA still finds a slot as the kernel before it drains, so all of them request
  // their weight tiles early (measured faster than two per SM on a 56-tile,
  // K = 16384 output projection); a short K would only add reduction work.
  int splits = 1;
  if (tiles > num_sms)
    splits = (8 * num_sms + tiles - 1) / tiles;
  else if (tiles > 0)
    splits = (2 * num_sms / tiles) * 16 <= num_kb ? (3 * num_sms / 2 + tiles - 1) / tiles : num_sms / tiles;
  const int max_splits = num_kb / 4 > 1 ? num_kb / 4 : 1;   // keep >= 4 K blocks per split
  splits = splits < 1 ? 1 : (splits > max_splits ? max_splits : splits);
  if (splits > 8) splits = 8;   // the splits of a tile form one (portable-size) cluster
  p.kb_per_split = (num_kb + splits - 1) / splits;
  p.splits = (num_kb + p.kb_per_split - 1) / p.kb_per_split;
  p.tiles = tiles;
  p.ws_bytes = 0;               // partials are reduced through distributed shared memory
  return p;
}

cudaError_t launch_gemm_bf16(const GemmArgs& a, bool swap, int bn, int token_tiles, cudaStream_t st,
                             const char* name) {
  dim3 grid(a.seg_tile_begin[a.n_seg], token_tiles, swap ? (a.splits > 1 ? a.splits : 1) : 1);
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  if (swap) {
    switch (bn) {
      case 16: return launch_one<16, true>(a, grid, st, name);
      case 32: return launch_one<32, true>(a, grid, st, name);
      case 64: return launch_one<64, true>(a, grid, st, name);
      case 128: return launch_one<128, true>(a, grid, st, name);
      case 256: return launch_one<256, true>(a, grid, st, name);
    }
  } else {
    switch (bn) {
      case 128: return launch_one<128, false>(a, grid, st, name);
      case 256: return launch_one<256, false>(a, grid, st, name);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace gmla
