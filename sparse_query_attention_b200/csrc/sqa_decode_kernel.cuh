// sqa_decode_kernel.cuh - Sparse Query Attention decoding against a key/value
// cache on sm_100a (split over the cache, then a combine pass).
//
// What it computes (per sequence b, new token i < n_new, query head h;
// j = h / G): token i sits at position p = len_b - n_new + i of a sequence
// whose first len_b keys/values are in the cache, and
//   O[b,i,h,:] = sum_{u <= p} softmax_u(scale <Q[b,i,h,:], K[b,u,j,:]>) V[b,u,j,:]
//   LSE[b,h,i] = log sum_{u <= p} exp(scale <Q[b,i,h,:], K[b,u,j,:]>)
// Autoregressive decoding is the memory-bound regime that the abstract of
// "Sparse Query Attention (SQA): ..." sets apart from training and
// full-sequence work: every step streams the whole cache once, and each
// key/value byte feeds only the G query heads of its group.  The kernel is
// therefore built to stream the cache at HBM speed; SQA's fewer query heads
// shrink its arithmetic, not its bytes.
//
// Work split.  One CTA = one cache chunk [s * chunk, min((s+1) * chunk, len_b))
// of one key/value head j for g query heads of the group (g = largest power
// of two dividing G) and all n_new tokens: rows r = i * g + gg of a 128-row
// tile (g * n_new <= 128; rows past that are padding whose results are never
// read).  Two CTAs fit on an SM (TMEM 256 columns, <= 97 KB shared memory
// each), so one CTA's softmax overlaps the other's tensor-core work and
// prologue.  With more than one chunk per sequence the CTA writes its
// normalised partial output and log2-sum-exp to a workspace and
// decode_combine_kernel merges the chunks; with one chunk it writes the
// result directly.
//
// Roles (8 warps): warp 0 lane 0 TMA (Q once, then K_i, V_i of 64 keys into
// a ring), warp 1 tcgen05.mma (S = Q K_i^T into TMEM, O += P V_i with P read
// from TMEM), warp 2 TMEM allocation, warps 4-7 softmax + epilogue for the
// 32-row quarters that hold real rows (the others idle).
#pragma once

#include "sqa_ptx.cuh"

namespace sqa {

constexpr unsigned int kStatusBadLength = 1u;  // == SQA_ERR_INVALID_ARG
constexpr float kDecRescaleThreshold = 8.0f;   // log2 units: rescale O only past 2^8 growth

template <int D>
struct DecCfg {
  static_assert(D == 16 || D == 32 || D == 64 || D == 128, "head dim");
  static constexpr int kBK = 64;                     // keys per step
  static constexpr int kRowElems = D < 64 ? D : 64;  // elements per swizzled smem row
  static constexpr int kRowBytes = kRowElems * 2;
  static constexpr int kChunks = D / kRowElems;
  static constexpr uint32_t kSwizzle = kRowBytes == 128 ? kSw128 : (kRowBytes == 64 ? kSw64 : kSw32);
  static constexpr int kQChunkBytes = 128 * kRowBytes;
  static constexpr int kQBytes = kChunks * kQChunkBytes;    // 128 x D query tile
  static constexpr int kKvChunkBytes = kBK * kRowBytes;
  static constexpr int kKvBytes = kChunks * kKvChunkBytes;  // 64 x D key or value tile
  static constexpr int kSlots = 4;                          // K/V ring entries
  // At least 80 KB so that no more than two CTAs share an SM: two CTAs use
  // all 512 TMEM columns.
  static constexpr int kSmemUsed = kQBytes + kSlots * kKvBytes + 1024;
  static constexpr int kSmemBytes = kSmemUsed > 80 * 1024 ? kSmemUsed : 80 * 1024;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColS = 0, kColO = 64;  // S: 64 fp32 columns (P over its first 32); O: D
  static_assert(kColO + D <= kTmemCols, "TMEM columns");
};

struct DecParams {
  void* out;              // final [B, n_new, H_q, D] (fp32 or bf16), when n_split == 1
  float* lse;             // final [B, H_q, n_new] (natural log) or null, when n_split == 1
  float* part_o;          // [n_split, B, n_new, H_q, D] fp32, when n_split > 1
  float* part_l;          // [n_split, B, n_new, H_q] log2-sum-exp, when n_split > 1
  const int* cache_lens;  // [B] valid cache tokens per sequence
  int B, n_new, H_q, H_kv, G, g, log2g, n_sub, L_max;
  int chunk, n_split;
  int out_bf16;
  float scale_log2;
};

constexpr int kDecThreads = 256;

// Valid cache length of sequence b, clamped into [n_new, L_max]; a value out
// of range sets the device status word (reported by sqa_device_status).
__device__ __forceinline__ int decode_len(const DecParams& p, int b, bool report) {
  int len = p.cache_lens[b];
  if (len < p.n_new || len > p.L_max) {
    if (report) atomicOr(&g_status_word, kStatusBadLength);
    len = len < p.n_new ? p.n_new : p.L_max;
  }
  return len;
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 2)
    sqa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  using C = DecCfg<D>;
  const int split = blockIdx.x;
  const int j = blockIdx.y / p.n_sub;
  const int sub = blockIdx.y % p.n_sub;
  const int b = blockIdx.z;
  // Programmatic dependent launch: the previous kernel on the stream (which
  // may have written the cache, the lengths or read this workspace) is
  // complete before anything touches global memory.
  grid_dependency_wait();
  const int len = decode_len(p, b, threadIdx.x == 0 && split == 0 && blockIdx.y == 0);
  const int kstart = split * p.chunk;
  if (kstart >= len) return;  // the whole CTA: this chunk lies past the sequence
  const int kend = min(kstart + p.chunk, len);
  const int n_steps = (kend - kstart + C::kBK - 1) / C::kBK;
  const int rows = p.g * p.n_new;             // real rows of the tile
  const int active_warps = (rows + 31) / 32;  // softmax warps with real rows
  const int h0 = j * p.G + sub * p.g;
  const int pos0 = len - p.n_new;  // position of new token 0

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t slot_full[C::kSlots];
  __shared__ __align__(8) uint64_t slot_empty[C::kSlots];
  __shared__ __align__(8) uint64_t s_full;
  __shared__ __align__(8) uint64_t p_ready;
  __shared__ __align__(8) uint64_t o_done;
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* ring = smem + C::kQBytes;
  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&p_ready, active_warps);
    mbar_init(&o_done, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ======================= TMA producer =================================
    if (lane == 0) {
      // Only the rows * row bytes the box covers arrive; the rest of the
      // 128-row tile is padding.
      mbar_arrive_expect_tx(&q_full, static_cast<uint32_t>(C::kChunks * rows * C::kRowBytes));
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(&tm_q, &q_full, q_smem + c * C::kQChunkBytes, c * C::kRowElems, h0, 0, b);
      int load = 0;  // ring position: K_0, V_0, K_1, V_1, ...
      bool ok = true;
      for (int i = 0; i < n_steps && ok; ++i) {
        for (int kv = 0; kv < 2; ++kv, ++load) {
          const int s = load % C::kSlots;
          if (load >= C::kSlots && !mbar_wait(&slot_empty[s], ((load / C::kSlots) - 1) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&slot_full[s], C::kKvBytes);
          uint8_t* dst = ring + s * C::kKvBytes;
          const CUtensorMap* m = kv == 0 ? &tm_k : &tm_v;
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(m, &slot_full[s], dst + c * C::kKvChunkBytes, c * C::kRowElems, j, kstart + i * C::kBK, b);
        }
      }
      // Every load of this CTA is issued: the combine pass may be scheduled
      // once all CTAs are here (it waits for this grid to finish anyway).
      grid_launch_dependents();
      mbar_drain(&q_full, 0);
      for (int l = max(0, load - C::kSlots); l < load; ++l) mbar_drain(&slot_full[l % C::kSlots], (l / C::kSlots) & 1);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (whole warp, lane 0 issues) ========
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::kBK, 0, 0);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
    const uint64_t q_kd = smem_desc(smem_addr(q_smem), 16, 8 * C::kRowBytes, C::kSwizzle);
    const uint64_t ring_kd = smem_desc(smem_addr(ring), 16, 8 * C::kRowBytes, C::kSwizzle);
    const uint64_t ring_mn = smem_desc(smem_addr(ring), C::kKvChunkBytes, 8 * C::kRowBytes, C::kSwizzle);
    bool ok = mbar_wait(&q_full, 0, &abort_flag);
    for (int i = 0; i < n_steps && ok; ++i) {
      const int kpos = 2 * i, vpos = 2 * i + 1;
      const int ks = kpos % C::kSlots, vs = vpos % C::kSlots;
      if (!mbar_wait(&slot_full[ks], (kpos / C::kSlots) & 1, &abort_flag)) break;
      tc_fence_after();
      // S = Q K_i^T.  S shares its TMEM columns with P of the previous step;
      // the tensor core runs this CTA's MMAs in issue order, so PV(i-1) has
      // read P before S(i) overwrites it.
      {
        const uint64_t b0 = desc_advance(ring_kd, ks * C::kKvBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          constexpr int kPerChunk = C::kRowElems / 16;
          const uint32_t qoff = (kk / kPerChunk) * C::kQChunkBytes + (kk % kPerChunk) * 32;
          const uint32_t koff = (kk / kPerChunk) * C::kKvChunkBytes + (kk % kPerChunk) * 32;
          mma_ss_w(tmem + C::kColS, desc_advance(q_kd, qoff), desc_advance(b0, koff), idesc_s, kk > 0);
        }
      }
      mma_commit_w(&s_full);
      mma_commit_w(&slot_empty[ks]);
      if (!mbar_wait(&slot_full[vs], (vpos / C::kSlots) & 1, &abort_flag)) break;
      // The tile holding the end of the sequence: cache rows past it are
      // in-bounds memory of any content (NaN included), and P = 0 there
      // would still give 0 * NaN in P V.  Zero those V rows (a row stays
      // inside its own 128/64/32-byte line under every swizzle mode).
      const int valid = kend - (kstart + i * C::kBK);
      if (valid < C::kBK) {
        uint8_t* vt = ring + vs * C::kKvBytes;
        const int n16 = (C::kBK - valid) * C::kRowBytes / 16;
        for (int c = 0; c < C::kChunks; ++c)
          for (int idx = lane; idx < n16; idx += 32)
            *reinterpret_cast<uint4*>(vt + c * C::kKvChunkBytes + valid * C::kRowBytes + idx * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (!mbar_wait(&p_ready, i & 1, &abort_flag)) break;
      tc_fence_after();
      {
        const uint64_t b0 = desc_advance(ring_mn, vs * C::kKvBytes);
#pragma unroll
        for (int kk = 0; kk < C::kBK / 16; ++kk)
          mma_ts_w(tmem + C::kColO, tmem + C::kColS + kk * 8, desc_advance(b0, kk * 16 * C::kRowBytes), idesc_o,
                   (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit_w(&o_done);
      mma_commit_w(&slot_empty[vs]);
    }
    mma_commit_w(&mma_done);
  } else if (warp >= 4 && warp - 4 < active_warps) {
    // ======================= softmax + epilogue ===========================
    const int wq = warp & 3;       // TMEM lane quarter
    const int r = wq * 32 + lane;  // tile row
    const bool real = r < rows;
    const int tok = r >> p.log2g;  // new token index
    const int head = h0 + (r & (p.g - 1));
    const int last_key = pos0 + tok;  // this row sees keys <= last_key
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + C::kColS;
    const uint32_t o_addr = lane_base + C::kColO;
    const float sl2 = p.scale_log2;
    // The tile's first masked key: chunk end, or the causal limit of token 0.
    const int mask_from = min(kend, pos0 + 1);

    float m_used = -INFINITY;  // running max (log2 units, scaled)
    float l_sum = 0.f;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      if (!mbar_wait(&s_full, i & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      const int key0 = kstart + i * C::kBK;
      float s[64];
      if (key0 + C::kBK > mask_from) {
        const int lim = min(kend, last_key + 1) - key0;  // columns [0, lim) are visible
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = c < lim ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]) * sl2;
      }
      float acc8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
      for (int c = 16; c < 64; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = fmax3(acc8[k], s[c + k], s[c + 8 + k]);
      const float mx =
          fmax3(fmax3(acc8[0], acc8[1], acc8[2]), fmax3(acc8[3], acc8[4], acc8[5]), fmaxf(acc8[6], acc8[7]));
      const float m_new = fmaxf(m_used, mx);
      const bool grow = m_new > m_used + kDecRescaleThreshold || (m_used == -INFINITY && m_new != -INFINITY);
      if (__any_sync(0xffffffffu, grow && i > 0 && m_used != -INFINITY)) {
        // O holds the steps before i once PV(i-1) has completed.
        if (!mbar_wait(&o_done, (i - 1) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
      uint32_t pk[32];
      float sum = 0.f;
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const float p0 = ex2_approx(s[2 * c2] - m_sub), p1 = ex2_approx(s[2 * c2 + 1] - m_sub);
        sum += p0 + p1;
        pk[c2] = pack_bf16x2(p0, p1);
      }
      l_sum += sum;
      tmem_st32(s_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready);
    }
    if (ok) ok = mbar_wait(&o_done, (n_steps - 1) & 1, &abort_flag);
    if (ok) {
      tc_fence_after();
      // A row that sees no key of this chunk (a later new token's chunk
      // starts past its position) contributes weight 0: O = 0, log-sum = -inf.
      const bool empty = !(l_sum > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l_sum;
      const size_t row = (static_cast<size_t>(b) * p.n_new + tok) * p.H_q + head;  // [b, tok, head]
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t orr[16];
        tmem_ld16(o_addr + c0, orr);
        tmem_wait_ld();
        if (real) {
          float v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(orr[c]) * inv_l;
          if (p.n_split > 1) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + (static_cast<size_t>(split) * p.B * p.n_new * p.H_q +
                                                                row) * D + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          } else if (p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row * D + c0);
            dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
            dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * D + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          }
        }
      }
      if (real) {
        const float l2 = empty ? -INFINITY : m_used + __log2f(l_sum);
        if (p.n_split > 1)
          p.part_l[static_cast<size_t>(split) * p.B * p.n_new * p.H_q + row] = l2;
        else if (p.lse != nullptr)
          p.lse[(static_cast<size_t>(b) * p.H_q + head) * p.n_new + tok] = l2 * 0.69314718055994531f;
      }
    }
  }

  // ---- teardown ------------------------------------------------------------
  __syncwarp();
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Merge of the per-chunk results: one 256-thread block per (b, token, head)
// row.  Its eight warps take the chunks in turn (warp w: chunks w, w + 8, ...),
// lane l holding columns [l * k, (l + 1) * k), k = max(1, D / 32) (at D = 16
// lanes 16-31 idle), so a row's chunks are read eight at a time rather than
// one after another; the warps' partial sums meet in shared memory.
//   M = max_s L_s,  w_s = 2^(L_s - M),  O = sum_s w_s O_s / sum_s w_s,
//   LSE = (M + log2 sum_s w_s) ln 2
// over the chunks s that start inside sequence b.
// ---------------------------------------------------------------------------
constexpr int kCombineWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) decode_combine_kernel(const DecParams p) {
  constexpr int kPer = D >= 32 ? D / 32 : 1;
  __shared__ float sm_acc[kCombineWarps][D];
  __shared__ float sm_w[kCombineWarps];
  const size_t n_rows = static_cast<size_t>(p.B) * p.n_new * p.H_q;
  const size_t row = blockIdx.x;  // grid = n_rows
  grid_dependency_wait();          // the partial results of the decode grid are complete
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = static_cast<int>(row % p.H_q);
  const int tok = static_cast<int>((row / p.H_q) % p.n_new);
  const int b = static_cast<int>(row / (static_cast<size_t>(p.H_q) * p.n_new));
  const int len = decode_len(p, b, false);
  const int n_used = (len + p.chunk - 1) / p.chunk;
  // Every warp forms the same M (same values, same order).
  float M = -INFINITY;
  for (int s = lane; s < n_used; s += 32) M = fmaxf(M, p.part_l[static_cast<size_t>(s) * n_rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  const bool on = lane * kPer < D;
#pragma unroll 2
  for (int s = warp; s < n_used; s += kCombineWarps) {
    const float ls = p.part_l[static_cast<size_t>(s) * n_rows + row];
    const float w = ls == -INFINITY ? 0.f : exp2f(ls - M);
    wsum += w;
    if (on) {
      const float* src = p.part_o + (static_cast<size_t>(s) * n_rows + row) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, src[e], acc[e]);
      }
    }
  }
  if (on) {
#pragma unroll
    for (int e = 0; e < kPer; ++e) sm_acc[warp][lane * kPer + e] = acc[e];
  }
  if (lane == 0) sm_w[warp] = wsum;
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float a = 0.f, wt = 0.f;
#pragma unroll
    for (int g = 0; g < kCombineWarps; ++g) {
      a += sm_acc[g][c];
      wt += sm_w[g];
    }
    const float v = a / wt;
    if (p.out_bf16)
      static_cast<__nv_bfloat16*>(p.out)[row * D + c] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(p.out)[row * D + c] = v;
    if (c == 0 && p.lse != nullptr)
      p.lse[(static_cast<size_t>(b) * p.H_q + head) * p.n_new + tok] = (M + __log2f(wt)) * 0.69314718055994531f;
  }
}

}  // namespace sqa
