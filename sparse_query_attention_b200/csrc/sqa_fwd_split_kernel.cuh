// sqa_fwd_split_kernel.cuh - SQA forward at d = 128 for grids too small to
// fill the GPU's waves.
//
// Computes exactly what sqa_fwd_kernel computes (the attention core of
// "Sparse Query Attention (SQA): A Computationally Efficient Attention
// Mechanism with Query Heads Reduction", abstract).  The two-tile kernel
// gives each CTA two 128-row query tiles; with few query heads (xSQA: 4
// heads of 32768 tokens) that is 512 CTAs, 3.5 waves on 148 SMs, and the
// last wave runs half empty.  Here each CTA takes ONE query tile and its two
// tiles (the two softmax warpgroups and their TMEM S/O pairs) take the
// even and the odd 128-key K/V blocks of that tile's key range: twice the
// CTAs, each with the same two-tile overlap of softmax and tensor-core work.
// The epilogue merges the two halves of every row by their running max and
// sum (m = max(m_a, m_b), l = l_a 2^(m_a - m) + l_b 2^(m_b - m),
// O = (O_a 2^(m_a - m) + O_b 2^(m_b - m)) / l), the merge any split of the
// key range admits.  Shared memory holds the one query tile and a five-slot
// K/V ring (each step loads four tiles: K and V of the even and the odd
// block).  Roles, TMEM layout, softmax and masking are those of the
// two-tile kernel.
#pragma once

#include "sqa_fwd_kernel.cuh"
#include "sqa_fwd_quad_kernel.cuh"  // named_bar_sync

namespace sqa {

template <int D>
struct SplitCfg {
  static_assert(D == 128, "the split kernel covers d = 128");
  using F = FwdCfg<D>;
  static constexpr int kRowElems = F::kRowElems;
  static constexpr int kRowBytes = F::kRowBytes;
  static constexpr int kChunks = F::kChunks;
  static constexpr int kChunkBytes = F::kChunkBytes;
  static constexpr int kTileBytes = F::kTileBytes;
  static constexpr uint32_t kSwizzle = F::kSwizzle;
  static constexpr int kSlots = 5;              // K/V ring entries
  static constexpr int kQBytes = kTileBytes;    // one query tile
  static constexpr int kSmemBytes = kQBytes + kSlots * kTileBytes + 1024;
  static constexpr uint32_t kTmemCols = F::kTmemCols;
  static constexpr uint32_t kColS0 = F::kColS0, kColS1 = F::kColS1, kColO0 = F::kColO0, kColO1 = F::kColO1;
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    sqa_fwd_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = SplitCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t slot_full[C::kSlots];
  __shared__ __align__(8) uint64_t slot_empty[C::kSlots];
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t p_ready[2][2];  // [tile][half of the keys]
  __shared__ __align__(8) uint64_t o_done[2];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ float merge_m[2][128];  // running max / sum per tile and row, for the merge
  __shared__ float merge_l[2][128];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;                   // [chunks][128 rows][row bytes]: the one query tile
  uint8_t* ring = smem + C::kQBytes;        // [slots][chunks][128 rows][row bytes]

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  // ---- work unit -----------------------------------------------------------
  const int T = 128 >> p.log2g;  // tokens per tile
  const BlockUnit u = block_unit(p.longest_first);
  const int tblk = p.tblk0 + (p.longest_first ? (p.n_tblk - 1 - u.x) : u.x);
  const int j = u.y / p.n_sub;
  const int sub = u.y % p.n_sub;
  const int b = u.z;
  const int h0 = j * p.G + sub * p.g;
  const int t0 = tblk * T;  // both tiles: tokens [t0, t0 + T)
  // KV blocks [blk_lo, blk_hi) hold every key a row of the query tile can
  // see; tile t takes blocks blk_lo + 2 i + t.  When the count is odd, tile
  // 1's last step lies past blk_hi and runs fully masked, so that the tiles
  // stay in lock-step with the MMA warp.
  int blk_lo, blk_hi;
  {
    const int tmax = min(t0 + T, p.N) - 1;
    const int lo = p.masked ? max(0, t0 - p.win_l) : 0;
    const int hi = p.masked ? min(p.Nkv, tmax + p.win_r + 1) : p.Nkv;
    blk_lo = lo / 128;
    blk_hi = (hi + 127) / 128;
  }
  const int n_steps = max(1, (blk_hi - blk_lo + 1) / 2);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_ready[t][0], 4);  // one arrival per softmax warp
      mbar_init(&p_ready[t][1], 4);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  // Programmatic dependent launch: the set-up above may overlap the end of
  // the previous kernel on the stream; nothing below touches global memory
  // before that kernel has completed.  Dependents are released only after
  // the barrier, once this CTA holds its TMEM: a dependent CTA that took the
  // SM's columns first would wait for this grid while this CTA waited for
  // the columns.
  // Exception (wait_at_exit): launched right after the two-tile kernel on the
  // other query tiles of the same problem, this grid reads only Q, K and V,
  // which the two-tile grid had already waited for before it released this
  // one, and writes rows that grid does not touch; so its CTAs start work at
  // once on the SMs that grid's last wave frees, and wait for that grid only
  // before they exit, so that this grid completes after it and the next
  // launch's wait covers both.
  if (!p.wait_at_exit) grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = tmem_base_sh;
  // Registers: the block launches with 384 x 168; the producer/MMA
  // warpgroup needs few, the two softmax warpgroups hold a 128-column score
  // row each: 88 * 128 + 208 * 256 = 168 * 384.  Each warpgroup reallocates
  // at the top of its own branch, so the register allocator sees which limit
  // governs which code.
  if (warp < 4) {
  regs_dealloc<kFwdRegsLow>();
  if (warp == 0) {
    // ======================= TMA producer =================================
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, C::kQBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(&tm_q, &q_full, q_smem + c * C::kChunkBytes, c * C::kRowElems, h0, t0, b);
      // Ring positions per step i: K of tile 0 and 1 (4i, 4i + 1), then V
      // of tile 0 and 1 (4i + 2, 4i + 3).  A block past the tensor reads as
      // zeros (TMA fill) and is masked.
      int load = 0;
      bool ok = true;
      for (int i = 0; i < n_steps && ok; ++i) {
        for (int u = 0; u < 4; ++u, ++load) {
          const int s = load % C::kSlots;
          if (load >= C::kSlots && !mbar_wait(&slot_empty[s], ((load / C::kSlots) - 1) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&slot_full[s], C::kTileBytes);
          uint8_t* dst = ring + s * C::kTileBytes;
          const CUtensorMap* m = u < 2 ? &tm_k : &tm_v;
          const int blk = blk_lo + 2 * i + (u & 1);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(m, &slot_full[s], dst + c * C::kChunkBytes, c * C::kRowElems, j, blk * 128, b);
        }
      }
      // Teardown: nothing may still be landing in shared memory at exit.
      mbar_drain(&q_full, 0);
      for (int l = max(0, load - C::kSlots); l < load; ++l) mbar_drain(&slot_full[l % C::kSlots], (l / C::kSlots) & 1);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ===================================
    // The whole warp runs this loop (warp-uniform values stay in uniform
    // registers, which keeps each tcgen05.mma issue short); lane 0 issues.
    {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t col_s[2] = {C::kColS0, C::kColS1};
      const uint32_t col_o[2] = {C::kColO0, C::kColO1};
      // Descriptors are built once; each MMA adds a constant offset.
      const uint64_t q_kd = smem_desc(smem_addr(q_smem), 16, 8 * C::kRowBytes, C::kSwizzle);
      const uint64_t ring_kd = smem_desc(smem_addr(ring), 16, 8 * C::kRowBytes, C::kSwizzle);
      const uint64_t ring_mn = smem_desc(smem_addr(ring), C::kChunkBytes, 8 * C::kRowBytes, C::kSwizzle);

      auto issue_s = [&](int t, int slot) {
        const uint64_t a0 = q_kd;  // both tiles hold the same query rows
        const uint64_t b0 = desc_advance(ring_kd, slot * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          constexpr int kPerChunk = C::kRowElems / 16;
          const uint32_t off = (kk / kPerChunk) * C::kChunkBytes + (kk % kPerChunk) * 32;
          mma_ss_w(tmem + col_s[t], desc_advance(a0, off), desc_advance(b0, off), idesc_s, kk > 0);
        }
      };
      // Four 16-key MMAs over keys [16 k0, 16 k0 + 64).
      auto issue_pv = [&](int t, int slot, bool acc, int k0) {
        const uint64_t b0 = desc_advance(ring_mn, slot * C::kTileBytes);
#pragma unroll
        for (int kk = k0; kk < k0 + 4; ++kk)
          mma_ts_w(tmem + col_o[t], tmem + col_s[t] + kk * 8, desc_advance(b0, kk * 16 * C::kRowBytes), idesc_o,
                 (acc || kk > k0) ? 1u : 0u);
      };

      bool ok = mbar_wait(&q_full, 0, &abort_flag);
      // Step 0 scores (ring positions 0 and 1).
      if (ok) ok = mbar_wait(&slot_full[0], 0, &abort_flag) && mbar_wait(&slot_full[1], 0, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit_w(&s_full[0]);
        mma_commit_w(&slot_empty[0]);
        issue_s(1, 1);
        mma_commit_w(&s_full[1]);
        mma_commit_w(&slot_empty[1]);
      }
      // Per step i, tile t: V at ring position 4i + 2 + t, the next K at
      // 4 (i + 1) + t.
      auto wait_pos = [&](int pos) { return mbar_wait(&slot_full[pos % C::kSlots], (pos / C::kSlots) & 1, &abort_flag); };
      for (int i = 0; i < n_steps && ok; ++i) {
        const int vpos0 = 4 * i + 2, kpos0 = 4 * i + 4;
        const bool more = i + 1 < n_steps;
        if (!wait_pos(vpos0) || !wait_pos(vpos0 + 1)) break;
        if (more && (!wait_pos(kpos0) || !wait_pos(kpos0 + 1))) break;
        int vs = vpos0 % C::kSlots, ks = kpos0 % C::kSlots;
        // tile 0: O_0 += P_0 V_i (keys 0-63 as soon as that half of P is
        // in TMEM, then keys 64-127), then S_0 = Q_0 K_{i+1}^T
        if (!mbar_wait(&p_ready[0][0], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(0, vs, i > 0, 0);
        if (!mbar_wait(&p_ready[0][1], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(0, vs, true, 4);
        if (!more) mma_commit_w(&o_done[0]);  // the epilogue's signal; S(i+1) carries it otherwise
        mma_commit_w(&slot_empty[vs]);
        if (more) {
          issue_s(0, ks);
          mma_commit_w(&s_full[0]);
          mma_commit_w(&slot_empty[ks]);
        }
        // tile 1: its own V and K slots
        vs = (vpos0 + 1) % C::kSlots;
        ks = (kpos0 + 1) % C::kSlots;
        if (!mbar_wait(&p_ready[1][0], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(1, vs, i > 0, 0);
        if (!mbar_wait(&p_ready[1][1], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(1, vs, true, 4);
        if (!more) mma_commit_w(&o_done[1]);
        mma_commit_w(&slot_empty[vs]);
        if (more) {
          issue_s(1, ks);
          mma_commit_w(&s_full[1]);
          mma_commit_w(&slot_empty[ks]);
        }
      }
      mma_commit_w(&mma_done);
    }
  }
  } else {
    regs_alloc<kFwdRegsHigh>();
    // ======================= softmax + epilogue ===========================
    const int t = (warp - 4) >> 2;  // tile
    const int wq = warp & 3;        // TMEM lane quarter
    const int r = wq * 32 + lane;   // row within the tile
    const int tok = t0 + (r >> p.log2g);  // the same rows in both tiles
    const int head = h0 + (r & (p.g - 1));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + (t == 0 ? C::kColS0 : C::kColS1);
    const uint32_t o_addr = lane_base + (t == 0 ? C::kColO0 : C::kColO1);
    const float sl2 = p.scale_log2;
    const int tile_tok_min = t0;
    const int tile_tok_max = min(tile_tok_min + T, p.N) - 1;
    // Both tiles step in lock-step with the MMA warp, n_steps each.

    float m_used = -INFINITY;  // running max in log2 units (of scaled scores)
    float l_sum = 0.f;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      if (!mbar_wait(&s_full[t], i & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      // Masking: keys past Nkv, keys outside the band, and whole tiles
      // outside this query tile's range.  Unmasked tiles (the common case)
      // keep raw scores: the row max is taken on them and the scale is
      // folded into the exponent's FFMA.  Masked tiles are scaled first and
      // get -inf where masked.
      const int kt = blk_lo + 2 * i + t;  // this tile's K/V block
      const int key0 = kt * 128;
      const bool outside = kt >= blk_hi;
      const bool need_mask = (key0 + 128 > p.Nkv) || outside ||
                             (p.masked && (key0 + 127 > tile_tok_min + p.win_r || key0 < tile_tok_max - p.win_l));
      float mult = sl2;  // exponent argument = s * mult - m
      if (need_mask) {
        int lo = 0, lim = p.Nkv - key0;  // columns [lo, lim) are visible
        if (p.masked) {
          lo = tok - p.win_l - key0;
          lim = min(lim, tok + p.win_r - key0 + 1);
        }
        if (outside) lim = 0;
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (c >= lo && c < lim) ? s[c] * sl2 : -INFINITY;
        mult = 1.f;
      }
      // Row max (row min for a negative scale on raw scores): eight
      // independent 3-input chains, then a short merge.  The sign test is a
      // uniform branch around whole loops, not a select per element.
      const bool use_min = !need_mask && sl2 < 0.f;
      float acc8[8];
      float ext;
      if (use_min) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = fminf(s[k], s[k + 8]);
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc8[k] = fmin3(acc8[k], s[c + k], s[c + 8 + k]);
        ext = fmin3(fmin3(acc8[0], acc8[1], acc8[2]), fmin3(acc8[3], acc8[4], acc8[5]), fminf(acc8[6], acc8[7]));
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc8[k] = fmax3(acc8[k], s[c + k], s[c + 8 + k]);
        ext = fmax3(fmax3(acc8[0], acc8[1], acc8[2]), fmax3(acc8[3], acc8[4], acc8[5]), fmaxf(acc8[6], acc8[7]));
      }
      const float mx = ext * mult;
      const float m_new = fmaxf(m_used, mx);
      // Rescale only when the running max grew by more than the threshold
      // (or on the first finite max); otherwise keep exponentiating against
      // the stale max, which bounds P by 2^8.
      const bool grow = m_new > m_used + kRescaleThreshold || (m_used == -INFINITY && m_new != -INFINITY);
      if (__any_sync(0xffffffffu, grow && i > 0 && m_used != -INFINITY)) {
        // O holds the sum over steps < i, and it is final: PV(i-1) was
        // issued before S(i), and the commit that signalled S(i) tracks
        // every earlier MMA of the issuing thread.
        const float f = (grow && m_used != -INFINITY) ? ex2_approx(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t orr[16];
          tmem_ld16(o_addr + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * f);
          tmem_st16(o_addr + c0, orr);
        }
        tmem_wait_st();
      }
      if (grow) {
        l_sum *= (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
      // P = 2^(s * mult - m): one packed FFMA per pair; every fourth pair on
      // the FMA pipe (polynomial), the rest on the MUFU; row sum in four
      // packed accumulators.  Keys 0-63 are stored and handed to the MMA
      // warp first, so the first half of O += P V runs while keys 64-127
      // are exponentiated.
      const uint64_t mult2 = f2_pack(mult, mult);
      const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int c = half * 32 + cc;
          float x0, x1, p0, p1;
          f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), mult2, negm2), x0, x1);
          if ((c & 3) == 3) {
            exp2_poly_pair(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          sum2[c & 3] = f2_add(sum2[c & 3], f2_pack(p0, p1));
          pk[cc] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_addr + half * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready[t][half]);
      }
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), a0, a1);
        l_sum += a0 + a1;
      }
    }
    // Epilogue: once the last PV of both tiles has landed, merge the two
    // halves of the key blocks by their running max and sum; tile t writes
    // columns [t d/2, (t + 1) d/2) and tile 0 the LSE.  Every softmax thread
    // reaches the named barrier, also after a timeout.
    if (ok) ok = mbar_wait(&o_done[t], 0, &abort_flag);  // committed once, after the last PV
    if (ok) ok = mbar_wait(&o_done[t ^ 1], 0, &abort_flag);
    merge_m[t][r] = m_used;
    merge_l[t][r] = l_sum;
    named_bar_sync(1, 256);
    if (ok) {
      tc_fence_after();
      const float ma = merge_m[0][r], la = merge_l[0][r];
      const float mb = merge_m[1][r], lb = merge_l[1][r];
      const float m = fmaxf(ma, mb);
      const float fa = ma == -INFINITY ? 0.f : ex2_approx(ma - m);
      const float fb = mb == -INFINITY ? 0.f : ex2_approx(mb - m);
      const float l = la * fa + lb * fb;
      const float inv_l = 1.f / l;
      const bool valid = tok < p.N;
      const size_t row_off = ((static_cast<size_t>(b) * p.N + (valid ? tok : 0)) * p.H_q + head) * D;
      const uint32_t oa = lane_base + C::kColO0, ob = lane_base + C::kColO1;
#pragma unroll 1
      for (int c0 = t * (D / 2); c0 < (t + 1) * (D / 2); c0 += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld16(oa + c0, ra);
        tmem_ld16(ob + c0, rb);
        tmem_wait_ld();
        if (valid) {
          float v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = (__uint_as_float(ra[c]) * fa + __uint_as_float(rb[c]) * fb) * inv_l;
          if (p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row_off + c0);
            dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
            dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row_off + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          }
        }
      }
      if (t == 0 && valid && p.lse != nullptr)
        p.lse[(static_cast<size_t>(b) * p.H_q + head) * p.N + tok] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  }

  // ---- teardown ------------------------------------------------------------
  __syncwarp();
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);  // every issued MMA has finished
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (p.wait_at_exit) grid_dependency_wait();
}

}  // namespace sqa
