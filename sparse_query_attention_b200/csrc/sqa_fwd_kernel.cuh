// sqa_fwd_kernel.cuh - fused Sparse Query Attention forward on sm_100a.
//
// What it computes (per batch b, query head h, query token t; j = h / G,
// G = H_q / H_kv):
//   O[b,t,h,:] = sum_u softmax_u(scale * <Q[b,t,h,:], K[b,u,j,:]>) V[b,u,j,:]
//   LSE[b,h,t] = log sum_u exp(scale * <Q[b,t,h,:], K[b,u,j,:]>)
// over the keys u visible to query t: all of them, or the band
// t - win_l <= u <= t + win_r (causal: win_l >= N, win_r = 0; a sliding
// window otherwise).  Only H_q query heads exist, so the two
// contractions cost 2 * B * H_q * P_c * d FLOPs each: the query-head
// reduction of "Sparse Query Attention (SQA): A Computationally Efficient
// Attention Mechanism with Query Heads Reduction" (abstract), built on the
// key/value sharing of Grouped Query Attention ("ReactiveAI/GQA-Ref-Micro"
// model card, introduction).
//
// Layout of the work.  One CTA owns two 128-row query tiles of ONE key/value
// head j.  A tile packs g query heads of the group side by side: row
// r = tt * g + gg is token t0 + tt, head h0 + gg (g = largest power of two
// dividing G, at most 128; 128 / g tokens per tile).  Every K/V tile is
// therefore fetched once by TMA and used by all the query heads the CTA
// holds -- the GQA/SQA sharing turned into on-chip reuse.
//
// Roles (12 warps):
//   warp 0 (one lane)  TMA: Q tiles once, then K_i, V_i into a ring of slots.
//   warp 1 (one lane)  tcgen05.mma issue:  S_t = Q_t K_i^T  (SMEM x SMEM ->
//                      TMEM fp32), O_t += P_t V_i (P from TMEM, V from SMEM).
//   warps 4-7, 8-11    softmax for tile 0 / tile 1, one thread per row:
//                      TMEM S -> registers, mask, online max/sum in the log2
//                      domain, P = 2^(s - m) as bf16 back into TMEM over S,
//                      rescale of O in TMEM when the running max grew by more
//                      than 2^8, and the epilogue O / l, LSE.
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1  (128, 128, d, d columns); P_t
// occupies the first 64 columns of S_t.
// MMA order per KV step i: PV_0(i), S_0(i+1), PV_1(i), S_1(i+1), so that the
// softmax of one tile overlaps the tensor-core work of the other.
#pragma once

#include "sqa_ptx.cuh"

namespace sqa {

template <int D>
struct FwdCfg {
  static_assert(D == 16 || D == 32 || D == 64 || D == 128, "head dim");
  static constexpr int kRowElems = D < 64 ? D : 64;  // elements per swizzled smem row
  static constexpr int kRowBytes = kRowElems * 2;    // 32, 64 or 128
  static constexpr int kChunks = D / kRowElems;      // 64-wide column chunks (1 or 2)
  static constexpr int kChunkBytes = 128 * kRowBytes;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // one 128 x D bf16 tile
  static constexpr uint32_t kSwizzle = kRowBytes == 128 ? kSw128 : (kRowBytes == 64 ? kSw64 : kSw32);
  static constexpr int kSlots = D == 128 ? 4 : 6;  // K/V ring entries
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kSmemBytes = kQBytes + kSlots * kTileBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  // Key split over a cluster: per row of both tiles, the unnormalised O
  // (padded rows, spread over the banks) and then (running max, sum) as one
  // 16-byte slot, staged over Q and the ring.
  static constexpr int kPartStride = D + 4;         // floats per staged O row
  static constexpr int kPartMl = 256 * kPartStride;  // float offset of the (m, l) slots
  static_assert(kPartMl * 4 + 256 * 16 <= kQBytes + kSlots * kTileBytes, "staged rows fit over Q and the ring");
};

struct FwdParams {
  void* out;       // [B, N, H_q, D], fp32 or bf16
  float* lse;      // [B, H_q, N] or null
  int B, N, H_q, H_kv, G, g, log2g;  // N: query tokens
  int Nkv;         // key/value tokens (N for self-attention; causal needs Nkv == N)
  int n_sub;       // G / g head sub-groups per KV head
  int n_tblk;      // token blocks of 2 * (128 / g) tokens
  int masked;      // band mask active (causal or sliding window)
  int win_l, win_r;  // band: t - win_l <= u <= t + win_r (both <= N)
  int longest_first;  // schedule token blocks from the last one
  int tblk0;          // first token block of this launch (a problem may be split over two launches)
  int wait_at_exit;   // second launch of a split problem: wait for the previous grid only before exiting
  int kv_splits;      // two-tile kernel: CTAs (a cluster) sharing one token block's key range; 1 = none
  int out_bf16;
  float scale_log2;  // scale * log2(e)
};

constexpr int kFwdThreads = 384;
constexpr int kFwdRegsLaunch = 168;  // per thread at launch (launch bounds 384 x 1)
constexpr int kFwdRegsLow = 88;      // producer / MMA warpgroup after reallocation
constexpr int kFwdRegsHigh = 208;    // each softmax warpgroup after reallocation
static_assert(kFwdRegsLow * 128 + kFwdRegsHigh * 256 <= kFwdRegsLaunch * kFwdThreads,
              "register split exceeds the launch pool");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only past 2^8 growth

// kKvSplit: the instantiation launched in clusters that split the key range
// (p.kv_splits > 1); the other one carries none of that code.
template <int D, bool kKvSplit = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    sqa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t slot_full[C::kSlots];
  __shared__ __align__(8) uint64_t slot_empty[C::kSlots];
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t p_ready[2][2];  // [tile][half of the keys]
  __shared__ __align__(8) uint64_t o_done[2];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;                   // [2][chunks][128 rows][row bytes]
  uint8_t* ring = smem + C::kQBytes;        // [slots][chunks][128 rows][row bytes]

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  // ---- work unit -----------------------------------------------------------
  const int T = 128 >> p.log2g;  // tokens per tile
  const BlockUnit u = block_unit(p.longest_first);
  // Few query tiles against many keys (unmasked): the key blocks of a token
  // block are split over a cluster of p.kv_splits CTAs, CTA `rank` taking a
  // contiguous share; each row's partial O, running max and sum are merged
  // through distributed shared memory at the end.
  const int splits = kKvSplit ? p.kv_splits : 1;
  const int rank = kKvSplit ? static_cast<int>(cluster_rank()) : 0;
  const int ux = kKvSplit ? u.x / splits : u.x;
  const int tblk = p.tblk0 + (p.longest_first ? (p.n_tblk - 1 - ux) : ux);
  const int j = u.y / p.n_sub;
  const int sub = u.y % p.n_sub;
  const int b = u.z;
  const int h0 = j * p.G + sub * p.g;
  const int t0 = tblk * 2 * T;  // tile 0 tokens [t0, t0+T), tile 1 [t0+T, t0+2T)
  // KV tiles [kv_lo[t], kv_hi[t]) hold every key a row of query tile t can
  // see; the CTA streams the union [kv_begin, kv_begin + n_steps).  Tile 0
  // always has tokens (t0 < N); a tile 1 entirely past N gets an empty range,
  // runs its steps fully masked so its barriers stay in lock-step, and
  // stores nothing.
  int kv_lo[2], kv_hi[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int tmin = t0 + t * T, tmax = min(t0 + (t + 1) * T, p.N) - 1;
    const int lo = p.masked ? max(0, tmin - p.win_l) : 0;
    const int hi = p.masked ? min(p.Nkv, tmax + p.win_r + 1) : p.Nkv;
    kv_lo[t] = lo / 128;
    kv_hi[t] = (hi + 127) / 128;
  }
  if constexpr (kKvSplit) {  // unmasked: both tiles see every key block
    const int nb = (p.Nkv + 127) / 128;
    kv_lo[0] = kv_lo[1] = static_cast<int>(static_cast<long long>(nb) * rank / splits);
    kv_hi[0] = kv_hi[1] = static_cast<int>(static_cast<long long>(nb) * (rank + 1) / splits);
  }
  const int kv_begin = kv_lo[0];
  if (t0 + T >= p.N) kv_lo[1] = kv_hi[1] = kv_begin;  // tile 1 holds no token
  const int n_steps = max(1, max(kv_hi[0], kv_hi[1]) - kv_begin);

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
  grid_dependency_wait();
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
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(&tm_q, &q_full, q_smem + (t * C::kChunks + c) * C::kChunkBytes, c * C::kRowElems, h0,
                      t0 + t * T, b);
      int load = 0;  // ring position: K_0, V_0, K_1, V_1, ...
      bool ok = true;
      for (int i = 0; i < n_steps && ok; ++i) {
        for (int kv = 0; kv < 2; ++kv, ++load) {
          const int s = load % C::kSlots;
          if (load >= C::kSlots && !mbar_wait(&slot_empty[s], ((load / C::kSlots) - 1) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&slot_full[s], C::kTileBytes);
          uint8_t* dst = ring + s * C::kTileBytes;
          const CUtensorMap* m = kv == 0 ? &tm_k : &tm_v;
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(m, &slot_full[s], dst + c * C::kChunkBytes, c * C::kRowElems, j, (kv_begin + i) * 128, b);
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
        const uint64_t a0 = desc_advance(q_kd, t * C::kTileBytes);
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
      // Step 0 scores.
      // Ring positions: K_i at 2i, V_i at 2i + 1.
      if (ok) ok = mbar_wait(&slot_full[0], 0, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit_w(&s_full[0]);
        issue_s(1, 0);
        mma_commit_w(&s_full[1]);
        mma_commit_w(&slot_empty[0]);
      }
      for (int i = 0; i < n_steps && ok; ++i) {
        const int vpos = 2 * i + 1, kpos = 2 * i + 2;
        const int vs = vpos % C::kSlots, ks = kpos % C::kSlots;
        if (!mbar_wait(&slot_full[vs], (vpos / C::kSlots) & 1, &abort_flag)) break;
        const bool more = i + 1 < n_steps;
        if (more && !mbar_wait(&slot_full[ks], (kpos / C::kSlots) & 1, &abort_flag)) break;
        // tile 0: O_0 += P_0 V_i (keys 0-63 as soon as that half of P is
        // in TMEM, then keys 64-127), then S_0 = Q_0 K_{i+1}^T
        if (!mbar_wait(&p_ready[0][0], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(0, vs, i > 0, 0);
        if (!mbar_wait(&p_ready[0][1], i & 1, &abort_flag)) break;
        tc_fence_after();
        issue_pv(0, vs, true, 4);
        if (!more) mma_commit_w(&o_done[0]);  // the epilogue's signal; S(i+1) carries it otherwise
        if (more) {
          issue_s(0, ks);
          mma_commit_w(&s_full[0]);
        }
        // tile 1
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
    const int tok = t0 + t * T + (r >> p.log2g);
    const int head = h0 + (r & (p.g - 1));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + (t == 0 ? C::kColS0 : C::kColS1);
    const uint32_t o_addr = lane_base + (t == 0 ? C::kColO0 : C::kColO1);
    const float sl2 = p.scale_log2;
    const int tile_tok_min = t0 + t * T;
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
      const int kt = kv_begin + i;
      const int key0 = kt * 128;
      const bool outside = kt < kv_lo[t] || kt >= kv_hi[t];
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
    // Epilogue: O / l and LSE once the last PV of this tile has landed.
    if (ok) ok = mbar_wait(&o_done[t], 0, &abort_flag);  // committed once, after the last PV
    if constexpr (kKvSplit) {
      // Stage the row's unnormalised O and its (running max, sum) over Q and
      // the ring, once no MMA of either tile reads them any more.
      if (ok) ok = mbar_wait(&mma_done, 0, &abort_flag);
      if (ok) {
        tc_fence_after();
        float* po = reinterpret_cast<float*>(smem) + (t * 128 + r) * C::kPartStride;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t orr[16];
          tmem_ld16(o_addr + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            reinterpret_cast<float4*>(po + c0)[q4] =
                make_float4(__uint_as_float(orr[4 * q4]), __uint_as_float(orr[4 * q4 + 1]),
                            __uint_as_float(orr[4 * q4 + 2]), __uint_as_float(orr[4 * q4 + 3]));
        }
        reinterpret_cast<float4*>(reinterpret_cast<float*>(smem) + C::kPartMl)[t * 128 + r] =
            make_float4(m_used, l_sum, 0.f, 0.f);
      }
    } else if (ok) {
      tc_fence_after();
      const bool valid = tok < p.N;
      const float inv_l = 1.f / l_sum;
      const size_t row_off = ((static_cast<size_t>(b) * p.N + (valid ? tok : 0)) * p.H_q + head) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t orr[16];
        tmem_ld16(o_addr + c0, orr);
        tmem_wait_ld();
        if (valid) {
          float v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(orr[c]) * inv_l;
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
      if (valid && p.lse != nullptr)
        p.lse[(static_cast<size_t>(b) * p.H_q + head) * p.N + tok] = (m_used + __log2f(l_sum)) * 0.69314718055994531f;
    }
  }

  __syncwarp();
  if constexpr (kKvSplit) {
    // Every CTA of the cluster has staged its rows (release / acquire at
    // cluster scope).  CTA `rank` merges rows [R0, R0 + nr) of the 256 (two
    // tiles) over the cluster in rank order:
    //   m = max_q m_q,  w_q = 2^(m_q - m),  l = sum_q w_q l_q,
    //   O = sum_q w_q O_q / l,  LSE = (m + log2 l) ln 2,
    // the merge a split of the key range admits; the second barrier keeps
    // every CTA's shared memory alive until all reads are done.
    cluster_sync();
    constexpr int kVec = D / 4;  // float4 per row
    const float* po = reinterpret_cast<const float*>(smem);
    const float4* pml = reinterpret_cast<const float4*>(po + C::kPartMl);
    const int rows = (256 + splits - 1) / splits;
    const int R0 = rank * rows;
    const int nr = max(0, min(256, R0 + rows) - R0);
    for (int item = threadIdx.x; item < nr * kVec; item += kFwdThreads) {
      const int R = R0 + item / kVec;
      const int c = (item % kVec) * 4;
      const int rr = R & 127;
      const int tok_r = t0 + (R >> 7) * T + (rr >> p.log2g);
      if (tok_r >= p.N) continue;
      const int head_r = h0 + (rr & (p.g - 1));
      float m = -INFINITY;
      for (int q = 0; q < splits; ++q) m = fmaxf(m, ld_cluster_f4(map_to_rank(pml + R, static_cast<uint32_t>(q))).x);
      float l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < splits; ++q) {
        const float4 ml = ld_cluster_f4(map_to_rank(pml + R, static_cast<uint32_t>(q)));
        const float w = ml.x == -INFINITY ? 0.f : ex2_approx(ml.x - m);
        l += ml.y * w;
        const float4 o = ld_cluster_f4(map_to_rank(po + R * C::kPartStride + c, static_cast<uint32_t>(q)));
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
      const float inv_l = 1.f / l;
      const size_t off = ((static_cast<size_t>(b) * p.N + tok_r) * p.H_q + head_r) * D + c;
      if (p.out_bf16) {
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + off) =
            make_uint2(pack_bf16x2(acc.x * inv_l, acc.y * inv_l), pack_bf16x2(acc.z * inv_l, acc.w * inv_l));
      } else {
        *reinterpret_cast<float4*>(static_cast<float*>(p.out) + off) =
            make_float4(acc.x * inv_l, acc.y * inv_l, acc.z * inv_l, acc.w * inv_l);
      }
      if (c == 0 && p.lse != nullptr)
        p.lse[(static_cast<size_t>(b) * p.H_q + head_r) * p.N + tok_r] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    cluster_sync();
  }

  // ---- teardown ------------------------------------------------------------
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);  // every issued MMA has finished
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace sqa
