// sqa_fwd_quad_kernel.cuh - SQA forward for head dims d <= 64 on sm_100a.
//
// Computes exactly what sqa_fwd_kernel computes (the attention core of
// "Sparse Query Attention (SQA): A Computationally Efficient Attention
// Mechanism with Query Heads Reduction", abstract: H_q < H query heads, each
// key/value head shared by G = H_q / H_kv of them), for d in {16, 32, 64}.
//
// Why a second kernel.  At d <= 64 the two contractions of a 128-key step
// are short next to the online softmax of 128 scores per row, so the kernel
// is bound by the softmax warps, and two of them per SM sub-partition (one
// per query tile) leave it latency-bound.  Here the CTA keeps the same two
// 128-row query tiles (so the grid, and how it fills the SMs, is unchanged)
// but splits every 128-key K/V block between two "virtual tiles" per query
// tile: keys 0-63 go to one, keys 64-127 to the other.  Four virtual tiles,
// four softmax warpgroups: twice the softmax warps per sub-partition, on
// 64-column rows.  Each virtual tile runs its own online softmax over its
// half of the keys; the epilogue merges the two halves of a query row by
// their running max and sum,
//   m = max(m_a, m_b),  l = l_a 2^(m_a - m) + l_b 2^(m_b - m),
//   O = (O_a 2^(m_a - m) + O_b 2^(m_b - m)) / l,  LSE = (m + log2 l) ln 2,
// the same merge a split of the key range always admits.  With four
// softmax warpgroups the single MMA-issuing warp becomes the limit: every
// tcgen05.mma costs ~55 cycles to issue whatever its size, and a step issues
// 32 small ones (N = 64); merging or splitting that issue was measured
// slower (one N = 128 score MMA per query tile couples the key halves; two
// issuing warps contend).
//
// Roles (20 warps):
//   warp 0 (one lane)  TMA: Q tiles once, then K_i, V_i into a ring of slots.
//   warp 1             tcgen05.mma issue (lane 0 issues, the warp runs the
//                      loop): S_v = Q_{v&1} K_i[half v>>1]^T (N = 64) and
//                      O_v += P_v V_i[half v>>1] (P from TMEM).
//   warps 4 + 4v ..    softmax of virtual tile v = 0..3 (query tile v & 1,
//                      key half v >> 1), one thread per row.
// TMEM (512 columns): S_v at 64 v (P_v over its first 32 columns as bf16
// pairs), O_v at 256 + 64 v.
#pragma once

#include "sqa_fwd_kernel.cuh"

namespace sqa {

constexpr int kQuadThreads = 640;
constexpr int kQuadRegsLaunch = 96;  // 65536 / 640 rounded down to a multiple of 8
constexpr int kQuadRegsLow = 56;     // producer / MMA warpgroup after reallocation
constexpr int kQuadRegsHigh = 104;   // each of the four softmax warpgroups
static_assert(kQuadRegsLow * 128 + kQuadRegsHigh * 512 <= kQuadRegsLaunch * kQuadThreads,
              "register split exceeds the launch pool");

template <int D>
struct QuadCfg {
  static_assert(D == 16 || D == 32 || D == 64, "the quad kernel covers d <= 64");
  using F = FwdCfg<D>;  // same shared-memory tiles and ring as the two-tile kernel
  static constexpr int kSlots = F::kSlots;
  static constexpr int kSmemBytes = F::kSmemBytes;
  static constexpr uint32_t kTmemCols = 512;
  __device__ static constexpr uint32_t col_s(int v) { return 64u * v; }
  __device__ static constexpr uint32_t col_o(int v) { return 256u + 64u * v; }
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kQuadThreads, 1)
    sqa_fwd_quad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = QuadCfg<D>;
  using F = typename C::F;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t slot_full[C::kSlots];
  __shared__ __align__(8) uint64_t slot_empty[C::kSlots];
  __shared__ __align__(8) uint64_t s_full[4];
  __shared__ __align__(8) uint64_t p_ready[4];
  __shared__ __align__(8) uint64_t o_done[4];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ float merge_m[4][128];  // running max / sum per virtual tile and row, for the merge
  __shared__ float merge_l[4][128];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;             // [2][128 rows][row bytes]
  uint8_t* ring = smem + F::kQBytes;  // [slots][128 rows][row bytes]

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  // ---- work unit (as in the two-tile kernel) --------------------------------
  const int T = 128 >> p.log2g;  // tokens per query tile
  const BlockUnit u = block_unit(p.longest_first);
  const int tblk = p.longest_first ? (p.n_tblk - 1 - u.x) : u.x;
  const int j = u.y / p.n_sub;
  const int sub = u.y % p.n_sub;
  const int b = u.z;
  const int h0 = j * p.G + sub * p.g;
  const int t0 = tblk * 2 * T;
  int kv_lo[2], kv_hi[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int tmin = t0 + t * T, tmax = min(t0 + (t + 1) * T, p.N) - 1;
    const int lo = p.masked ? max(0, tmin - p.win_l) : 0;
    const int hi = p.masked ? min(p.Nkv, tmax + p.win_r + 1) : p.Nkv;
    kv_lo[t] = lo / 128;
    kv_hi[t] = (hi + 127) / 128;
  }
  const int kv_begin = kv_lo[0];
  if (t0 + T >= p.N) kv_lo[1] = kv_hi[1] = kv_begin;  // query tile 1 holds no token
  const int n_steps = max(1, max(kv_hi[0], kv_hi[1]) - kv_begin);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int v = 0; v < 4; ++v) {
      mbar_init(&s_full[v], 1);
      mbar_init(&p_ready[v], 4);  // one arrival per softmax warp
      mbar_init(&o_done[v], 1);
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
  // Registers: 640 x 96 at launch; 56 x 128 + 104 x 512 after reallocation.
  if (warp < 4) {
  regs_dealloc<kQuadRegsLow>();
  if (warp == 0) {
    // ======================= TMA producer =================================
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, F::kQBytes);
      for (int t = 0; t < 2; ++t)
        tma_load_4d(&tm_q, &q_full, q_smem + t * F::kTileBytes, 0, h0, t0 + t * T, b);
      int load = 0;  // ring position: K_0, V_0, K_1, V_1, ...
      bool ok = true;
      for (int i = 0; i < n_steps && ok; ++i) {
        for (int kv = 0; kv < 2; ++kv, ++load) {
          const int s = load % C::kSlots;
          if (load >= C::kSlots && !mbar_wait(&slot_empty[s], ((load / C::kSlots) - 1) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&slot_full[s], F::kTileBytes);
          tma_load_4d(kv == 0 ? &tm_k : &tm_v, &slot_full[s], ring + s * F::kTileBytes, 0, j, (kv_begin + i) * 128, b);
        }
      }
      // Teardown: nothing may still be landing in shared memory at exit.
      mbar_drain(&q_full, 0);
      for (int l = max(0, load - C::kSlots); l < load; ++l) mbar_drain(&slot_full[l % C::kSlots], (l / C::kSlots) & 1);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ===================================
    // The whole warp runs this loop; lane 0 issues each tcgen05.mma.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // 128 rows x 64 keys
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);   // 128 rows x d, V MN-major
    // Descriptors built once; each MMA adds a constant offset.  Key half h
    // of a K or V tile starts 64 rows (a whole number of swizzle periods)
    // into the slot.
    const uint64_t q_kd = smem_desc(smem_addr(q_smem), 16, 8 * F::kRowBytes, F::kSwizzle);
    const uint64_t ring_kd = smem_desc(smem_addr(ring), 16, 8 * F::kRowBytes, F::kSwizzle);
    const uint64_t ring_mn = smem_desc(smem_addr(ring), F::kChunkBytes, 8 * F::kRowBytes, F::kSwizzle);
    auto issue_s = [&](int v, int slot) {
      const uint64_t a0 = desc_advance(q_kd, (v & 1) * F::kTileBytes);
      const uint64_t b0 = desc_advance(ring_kd, slot * F::kTileBytes + (v >> 1) * 64 * F::kRowBytes);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss_w(tmem + C::col_s(v), desc_advance(a0, kk * 32), desc_advance(b0, kk * 32), idesc_s, kk > 0);
    };
    // O_v += P_v V_i[half]: four 16-key MMAs, P_v from TMEM.
    auto issue_pv = [&](int v, int slot, bool acc) {
      const uint64_t b0 = desc_advance(ring_mn, slot * F::kTileBytes + (v >> 1) * 64 * F::kRowBytes);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts_w(tmem + C::col_o(v), tmem + C::col_s(v) + kk * 8, desc_advance(b0, kk * 16 * F::kRowBytes), idesc_o,
                 (acc || kk > 0) ? 1u : 0u);
    };

    bool ok = mbar_wait(&q_full, 0, &abort_flag);
    if (ok) ok = mbar_wait(&slot_full[0], 0, &abort_flag);
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        issue_s(v, 0);
        mma_commit_w(&s_full[v]);
      }
      mma_commit_w(&slot_empty[0]);
    }
    // Per KV step i: for each virtual tile, O_v += P_v V_i as soon as its
    // softmax has stored P_v, then S_v = Q K_{i+1}^T into the same columns.
    for (int i = 0; i < n_steps && ok; ++i) {
      const int vpos = 2 * i + 1, kpos = 2 * i + 2;
      const int vs = vpos % C::kSlots, ks = kpos % C::kSlots;
      if (!mbar_wait(&slot_full[vs], (vpos / C::kSlots) & 1, &abort_flag)) break;
      const bool more = i + 1 < n_steps;
      if (more && !mbar_wait(&slot_full[ks], (kpos / C::kSlots) & 1, &abort_flag)) break;
      bool good = true;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        if (!mbar_wait(&p_ready[v], i & 1, &abort_flag)) {
          good = false;
          break;
        }
        tc_fence_after();
        issue_pv(v, vs, i > 0);
        if (!more) mma_commit_w(&o_done[v]);  // the epilogue's signal; S(i+1) carries it otherwise
        if (more) {
          issue_s(v, ks);
          mma_commit_w(&s_full[v]);
        }
      }
      if (!good) break;
      mma_commit_w(&slot_empty[vs]);
      if (more) mma_commit_w(&slot_empty[ks]);
    }
    mma_commit_w(&mma_done);
  }
  } else {
    regs_alloc<kQuadRegsHigh>();
    // ======================= softmax + epilogue ===========================
    const int v = (warp - 4) >> 2;  // virtual tile
    const int qt = v & 1;           // query tile
    const int half = v >> 1;        // key half of every K/V block
    const int wq = warp & 3;        // TMEM lane quarter
    const int r = wq * 32 + lane;   // row within the tile
    const int tok = t0 + qt * T + (r >> p.log2g);
    const int head = h0 + (r & (p.g - 1));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + C::col_s(v);
    const uint32_t o_addr = lane_base + C::col_o(v);
    const float sl2 = p.scale_log2;
    const int tile_tok_min = t0 + qt * T;
    const int tile_tok_max = min(tile_tok_min + T, p.N) - 1;

    float m_used = -INFINITY;  // running max in log2 units (of scaled scores)
    float l_sum = 0.f;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      if (!mbar_wait(&s_full[v], i & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
      // Masking as in the two-tile kernel, over keys [key0, key0 + 64).
      const int kt = kv_begin + i;
      const int key0 = kt * 128 + half * 64;
      const bool outside = kt < kv_lo[qt] || kt >= kv_hi[qt];
      const bool need_mask = (key0 + 64 > p.Nkv) || outside ||
                             (p.masked && (key0 + 63 > tile_tok_min + p.win_r || key0 < tile_tok_max - p.win_l));
      float mult = sl2;  // exponent argument = s * mult - m
      if (need_mask) {
        int lo = 0, lim = p.Nkv - key0;  // columns [lo, lim) are visible
        if (p.masked) {
          lo = tok - p.win_l - key0;
          lim = min(lim, tok + p.win_r - key0 + 1);
        }
        if (outside) lim = 0;
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = (c >= lo && c < lim) ? s[c] * sl2 : -INFINITY;
        mult = 1.f;
      }
      // Row max (row min for a negative scale on raw scores): eight
      // independent 3-input chains, then a short merge.
      const bool use_min = !need_mask && sl2 < 0.f;
      float acc8[8];
      float ext;
      if (use_min) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = fminf(s[k], s[k + 8]);
#pragma unroll
        for (int c = 16; c < 64; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc8[k] = fmin3(acc8[k], s[c + k], s[c + 8 + k]);
        ext = fmin3(fmin3(acc8[0], acc8[1], acc8[2]), fmin3(acc8[3], acc8[4], acc8[5]), fminf(acc8[6], acc8[7]));
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
        for (int c = 16; c < 64; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc8[k] = fmax3(acc8[k], s[c + k], s[c + 8 + k]);
        ext = fmax3(fmax3(acc8[0], acc8[1], acc8[2]), fmax3(acc8[3], acc8[4], acc8[5]), fmaxf(acc8[6], acc8[7]));
      }
      const float mx = ext * mult;
      const float m_new = fmaxf(m_used, mx);
      // Rescale only when the running max grew by more than the threshold
      // (or on the first finite max), which bounds P by 2^8.
      const bool grow = m_new > m_used + kRescaleThreshold || (m_used == -INFINITY && m_new != -INFINITY);
      if (__any_sync(0xffffffffu, grow && i > 0 && m_used != -INFINITY)) {
        // O_v holds the sum over steps < i, and it is final: PV(i-1) was
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
      // P = 2^(s * mult - m): one packed FFMA per pair, every fourth pair on
      // the FMA pipe (polynomial), the rest on the MUFU; row sum in four
      // packed accumulators; P as bf16 pairs over the first 32 columns of S.
      const uint64_t mult2 = f2_pack(mult, mult);
      const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float x0, x1, p0, p1;
        f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), mult2, negm2), x0, x1);
        if ((c & 3) == 3) {
          exp2_poly_pair(x0, x1, p0, p1);
        } else {
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        sum2[c & 3] = f2_add(sum2[c & 3], f2_pack(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
      }
      tmem_st32(s_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[v]);
      float a0, a1;
      f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), a0, a1);
      l_sum += a0 + a1;
    }
    // Epilogue: once the last O += P V of both key halves of these rows has
    // landed, merge the halves by their running max and sum; half 0 writes
    // columns [0, d/2) and the LSE, half 1 columns [d/2, d) (half 0 alone at
    // d = 16).  Every thread of the query tile reaches the named barrier,
    // also after a timeout, so none is left waiting there.
    if (ok) ok = mbar_wait(&o_done[v], 0, &abort_flag);  // committed once, after the last PV
    if (ok) ok = mbar_wait(&o_done[v ^ 2], 0, &abort_flag);
    merge_m[v][r] = m_used;
    merge_l[v][r] = l_sum;
    named_bar_sync(1 + qt, 256);
    if (ok) {
      tc_fence_after();
      const float ma = merge_m[qt][r], la = merge_l[qt][r];
      const float mb = merge_m[qt + 2][r], lb = merge_l[qt + 2][r];
      const float m = fmaxf(ma, mb);
      const float fa = ma == -INFINITY ? 0.f : ex2_approx(ma - m);
      const float fb = mb == -INFINITY ? 0.f : ex2_approx(mb - m);
      const float l = la * fa + lb * fb;
      const float inv_l = 1.f / l;
      const bool valid = tok < p.N;
      const size_t row_off = ((static_cast<size_t>(b) * p.N + (valid ? tok : 0)) * p.H_q + head) * D;
      constexpr int kCols = D >= 32 ? D / 2 : D;
      const uint32_t oa = lane_base + C::col_o(qt), ob = lane_base + C::col_o(qt + 2);
#pragma unroll 1
      for (int c0 = half * kCols; c0 < (half + 1) * kCols && c0 < D; c0 += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld16(oa + c0, ra);
        tmem_ld16(ob + c0, rb);
        tmem_wait_ld();
        if (valid) {
          float o[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            o[c] = (__uint_as_float(ra[c]) * fa + __uint_as_float(rb[c]) * fb) * inv_l;
          if (p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row_off + c0);
            dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                pack_bf16x2(o[6], o[7]));
            dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                                pack_bf16x2(o[14], o[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row_off + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
          }
        }
      }
      if (half == 0 && valid && p.lse != nullptr)
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
}

}  // namespace sqa
