// sqa_bwd_kernel.cuh - gradient of the Sparse Query Attention core on sm_100a.
//
// With P_tu = exp(s_tu - LSE_t), s_tu = scale <q_t, k_u>, D_t = <dO_t, O_t>:
//   dV_j = sum_{h in group j} P^T dO_h
//   dS   = P o (dO_h V_j^T - D)
//   dQ_h = scale dS K_j
//   dK_j = scale sum_{h in group j} dS^T Q_h
// P is zero outside the visible keys: all keys, or the band
// t - win_l <= u <= t + win_r (causal, or a sliding window).
// The training-time gains the pages report ("ReactiveAI/GQA-Ref-Micro" model
// card, results; "Sparse Query Attention (SQA): ...", abstract: pre-training
// and fine-tuning) come from these contractions also running over H_q heads
// only.
//
// Three kernels, all launched on one stream, no atomics (deterministic):
//   bwd_prep_kernel   D_t and LSE_t * log2(e) into a padded fp32 workspace.
//   bwd_dkdv_kernel   KV-outer: one CTA per 128-key tile of one KV head; the
//                     keys are the TMEM lanes and the loop runs over every
//                     query head of the group and every 64-token query
//                     sub-tile, so the group sum of dK/dV happens inside one
//                     TMEM accumulator.  Per step: S^T = K Q^T and
//                     dP^T = V dO^T (tcgen05, SMEM x SMEM), softmax warps form
//                     P^T and dS^T in bf16 back in TMEM, then dV += P^T dO and
//                     dK += dS^T Q (A operand from TMEM).
//   bwd_dq_kernel     Q-outer: one CTA per 128 packed query rows (as in the
//                     forward); per 64-key sub-tile: S = Q K^T, dP = dO V^T,
//                     dS in TMEM, dQ += dS K.
// Score tiles are 64 wide and held in two or three TMEM buffers (three where
// the columns allow): the scores of step s + buffers are computed as soon as
// step s's products have read its buffer, so the softmax warps, which take
// steps in turn, find their scores ready.
#pragma once

#include "sqa_ptx.cuh"

namespace sqa {

// ---------------------------------------------------------------------------
// Preprocess: D[b,h,t] = sum_c dO[b,t,h,c] O[b,t,h,c]; L2[b,h,t] = LSE * log2 e,
// both stored negated.  Workspace rows are padded to n_pad tokens (multiple of
// 128) with zeros.
// HBM-bound: kLanes = D / 8 lanes per row, each reading 8 consecutive
// elements of O (fp32: two 16-byte loads; bf16: one) and of dO (one 16-byte
// load), so a warp covers 256 / D rows with fully used 16-byte accesses.
// ---------------------------------------------------------------------------
template <int D>
__global__ void bwd_prep_kernel(const void* __restrict__ o, int o_bf16, const __nv_bfloat16* __restrict__ dout,
                                const float* __restrict__ lse, float* __restrict__ dsum, float* __restrict__ lse2,
                                int B, int N, int H_q, int n_pad) {
  constexpr int kLanes = D / 8;  // 2 .. 16 lanes per row
  grid_dependency_wait();  // O and LSE of the previous kernel on the stream are complete
  grid_launch_dependents();
  const size_t gtid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t idx = gtid / kLanes;  // row of the padded [B, H_q, n_pad] space
  const int sub = static_cast<int>(gtid % kLanes);
  const size_t total = static_cast<size_t>(B) * H_q * n_pad;
  const bool in = idx < total;
  const int t = in ? static_cast<int>(idx % n_pad) : 0;
  const size_t bh = in ? idx / n_pad : 0;
  const int h = static_cast<int>(bh % H_q);
  const int b = static_cast<int>(bh / H_q);
  float acc = 0.f, l2 = 0.f;
  if (in && t < N) {
    const size_t base = ((static_cast<size_t>(b) * N + t) * H_q + h) * D + sub * 8;
    const uint4 g = *reinterpret_cast<const uint4*>(dout + base);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
    float ov[8];
    if (o_bf16) {
      const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + base);
      const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(u2[k]);
        ov[2 * k] = f.x;
        ov[2 * k + 1] = f.y;
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(o) + base);
      const float4 a = src[0], c = src[1];
      ov[0] = a.x, ov[1] = a.y, ov[2] = a.z, ov[3] = a.w, ov[4] = c.x, ov[5] = c.y, ov[6] = c.z, ov[7] = c.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(g2[k]);
      acc = fmaf(ov[2 * k], f.x, acc);
      acc = fmaf(ov[2 * k + 1], f.y, acc);
    }
    l2 = lse[bh * N + t] * 1.4426950408889634f;
  }
#pragma unroll
  for (int s = kLanes / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (in && sub == 0) {  // stored negated: the kernels add them in packed FFMA/FADD
    dsum[idx] = -acc;
    lse2[idx] = -l2;
  }
}

template <typename T>
__device__ __forceinline__ void store16(T* dst, const float (&v)[16]);
template <>
__device__ __forceinline__ void store16<float>(float* dst, const float (&v)[16]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[16]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  d4[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]));
  d4[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                     pack_bf16x2(v[14], v[15]));
}

template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

// Swizzled-tile geometry shared by the backward kernels: R rows of D bf16,
// stored as D/64 column chunks of R rows x (up to) 128 bytes.
template <int D, int R>
struct TileGeo {
  static constexpr int kRowElems = D < 64 ? D : 64;
  static constexpr int kRowBytes = kRowElems * 2;
  static constexpr int kChunks = D / kRowElems;
  static constexpr int kChunkBytes = R * kRowBytes;
  static constexpr int kBytes = kChunks * kChunkBytes;
  static constexpr uint32_t kSwizzle = kRowBytes == 128 ? kSw128 : (kRowBytes == 64 ? kSw64 : kSw32);
  static constexpr uint32_t kSbo = 8 * kRowBytes;

  // K-major operand (rows = M or N, K = D): base descriptor of a tile, and
  // the byte offset of the 16-wide K step kk within it.
  __device__ static uint64_t kmajor_base(uint32_t base) { return smem_desc(base, 16, kSbo, kSwizzle); }
  __host__ __device__ static constexpr uint32_t kmajor_off(int kk) {
    return ((kk * 16) / kRowElems) * kChunkBytes + ((kk * 16) % kRowElems) * 2;
  }
  // MN-major operand (N = D along the row, K = rows): base descriptor, and
  // the byte offset of rows [16 kk, 16 kk + 16).
  __device__ static uint64_t mnmajor_base(uint32_t base) { return smem_desc(base, kChunkBytes, kSbo, kSwizzle); }
  __host__ __device__ static constexpr uint32_t mnmajor_off(int kk) { return kk * 16 * kRowBytes; }
};

struct BwdParams {
  void* dq;
  void* dk;
  void* dv;
  const float* dsum;  // [B, H_q, n_pad]
  const float* lse2;  // [B, H_q, n_pad]
  int B, N, H_q, H_kv, G, n_pad;  // N: query tokens, n_pad: N rounded up to 128
  int Nkv;                        // key/value tokens (N for self-attention)
  int ld_dq, ld_dkv;              // token strides (elements) of dQ and of dK/dV
  int g, log2g, n_sub, n_tblk;  // packing of the dQ kernel
  int masked;                   // band mask active (causal or sliding window)
  int win_l, win_r;             // band: t - win_l <= u <= t + win_r (both <= N)
  int longest_first;            // causal: hand out the longest tiles first over the whole grid
  int kv_splits;                // dK/dV: CTAs (a cluster) sharing one key tile's steps; 1 = none
  int wait_at_exit;             // dQ launched right after dK/dV: wait for that grid only before exiting
  float scale;
  float scale_log2;
};

constexpr int kBwdThreads = 384;
// Register split after launch (384 x 168): producer/MMA warpgroup 104, the two
// softmax-gradient warpgroups 200 each; 104 * 128 + 200 * 256 = 168 * 384.
constexpr int kBwdRegsLow = 104;
constexpr int kBwdRegsHigh = 200;
static_assert(kBwdRegsLow * 128 + kBwdRegsHigh * 256 <= 168 * kBwdThreads, "register split exceeds the launch pool");

// ===========================================================================
// dK / dV
// ===========================================================================
template <int D>
struct DkdvCfg {
  using KV = TileGeo<D, 128>;  // resident K and V tiles
  using QT = TileGeo<D, 64>;   // streamed Q / dO sub-tiles
  static constexpr int kStages = D == 128 ? 4 : 6;
  // Per-query statistics folded into the score MMAs: a 16-wide K step whose
  // A operand is 1 in columns 0-2 for every key and whose B operand holds,
  // per query, -L2 / (scale log2 e) (resp. -D) split into three bf16 parts,
  // so S^T and dP^T arrive from the tensor core already shifted.  Both
  // operands use the unswizzled K-major layout: 8-row x 16-byte core
  // matrices, K neighbours 128 B apart, 8-row groups 256 B apart.
  static constexpr int kAugRowBytes = 32;                 // 16 bf16 per row
  static constexpr int kAugBytes = 64 * kAugRowBytes;     // one 64-query operand
  static constexpr int kOnesBytes = 128 * kAugRowBytes;   // the 128-key ones operand
  static constexpr int kStatLse = 0, kStatD = 256;        // fp32 -L2, -D (TMA)
  static constexpr int kStatAugL = 1024, kStatAugD = 1024 + kAugBytes;
  static constexpr int kStatBytes = 1024 + 2 * kAugBytes;            // 5 KB, keeps stages 1 KB aligned
  static constexpr int kStageBytes = 2 * QT::kBytes + kStatBytes;     // Q, dO, statistics
  static constexpr int kSmemBytes = 2 * KV::kBytes + kStages * kStageBytes + kOnesBytes + 1024;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  __host__ __device__ static constexpr uint32_t aug_off(int r, int e) {  // byte offset of element (r, e)
    return (r / 8) * 256 + (e / 8) * 128 + (r % 8) * 16 + (e % 8) * 2;
  }
  // Score buffers in TMEM: three when they fit next to dV and dK (d <= 64).
  static constexpr int kBufs = D <= 64 ? 3 : 2;
  // TMEM columns: S^T/P^T and dP^T/dS^T of buffer b, then dV and dK.
  __device__ static constexpr uint32_t col_s(int b) { return 128u * b; }
  __device__ static constexpr uint32_t col_dp(int b) { return 64u + 128u * b; }
  static constexpr uint32_t kColDV = 128 * kBufs, kColDK = 128 * kBufs + D;
  static_assert(kColDK + D <= 512, "TMEM columns");
  // Split over a cluster: partial dV and dK rows staged over the ring.
  static constexpr int kPartStride = D + 4;  // floats per row; the pad spreads rows over the banks
  static_assert(2 * 128 * kPartStride * 4 <= kStages * kStageBytes, "partial dV / dK fit over the ring");
};

// Splits v into three bf16 parts whose sum is v to about 2^-24 relative.
__device__ __forceinline__ void split3_bf16(float v, __nv_bfloat16& h, __nv_bfloat16& m, __nv_bfloat16& l) {
  h = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h);
  m = __float2bfloat16_rn(r1);
  l = __float2bfloat16_rn(r1 - __bfloat162float(m));
}

// kAug: statistics folded into the score MMAs (needs a scale with a finite
// 1 / (scale log2 e)); otherwise the softmax warps read them per column.
// kKvSplit: the instantiation launched in clusters that split each key
// tile's steps (p.kv_splits > 1); the other one carries none of that code.
template <int D, typename GradT, bool kAug, bool kKvSplit = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_lse2, const __grid_constant__ CUtensorMap tm_dsum,
                    const BwdParams p) {
  using C = DkdvCfg<D>;
  using KV = typename C::KV;
  using QT = typename C::QT;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t kv_full;
  __shared__ __align__(8) uint64_t st_full[C::kStages];
  __shared__ __align__(8) uint64_t st_empty[C::kStages];
  __shared__ __align__(8) uint64_t aug_full[C::kStages];
  __shared__ __align__(8) uint64_t s_full[C::kBufs];
  __shared__ __align__(8) uint64_t p_ready[C::kBufs];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* k_smem = smem;
  uint8_t* v_smem = smem + KV::kBytes;
  uint8_t* stages = smem + 2 * KV::kBytes;
  uint8_t* ones_smem = stages + C::kStages * C::kStageBytes;

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  // Causal: key tile 0 sees every query, so ascending tiles are longest first.
  const BlockUnit u = block_unit(p.longest_first);
  // Unmasked problems with few key tiles (cross / memory attention over a
  // short key sequence) split each key tile's steps over a cluster of
  // p.kv_splits CTAs: CTA `rank` takes a contiguous share of the
  // (query head, query sub-tile) steps, and the partial dK / dV are summed
  // through distributed shared memory at the end.
  const int splits = kKvSplit ? p.kv_splits : 1;
  const int rank = kKvSplit ? static_cast<int>(cluster_rank()) : 0;
  const int kt = kKvSplit ? u.x / splits : u.x;  // key tile
  const int j = u.y;
  const int b = u.z;
  const int key0 = kt * 128;
  // Queries that can see a key of this tile: t in [key0 - win_r,
  // key0 + 127 + win_l] within [0, N); streamed as 64-token sub-tiles.
  const int q_lo = p.masked ? max(0, key0 - p.win_r) : 0;
  const int q_hi = p.masked ? min(p.N, key0 + 128 + p.win_l) : p.N;
  const int qs_begin = q_lo / 64;
  const int per_head = max(0, (q_hi + 63) / 64 - qs_begin);
  const int n_all = p.G * per_head;  // steps of this key tile; this CTA runs [s_begin, s_begin + n_steps)
  const int s_begin = static_cast<int>(static_cast<long long>(n_all) * rank / splits);
  const int n_steps = static_cast<int>(static_cast<long long>(n_all) * (rank + 1) / splits) - s_begin;

  if (threadIdx.x == 0) {
    mbar_init(&kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
      mbar_init(&aug_full[s], 1);
    }
    for (int t = 0; t < C::kBufs; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_ready[t], 4);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
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

  if (warp < 4) {
  regs_dealloc<kBwdRegsLow>();
  if (kAug && warp == 3) {
    // ---------------- statistics operands (whole warp) ----------------
    // The ones operand once, then per stage the three-part bf16 split of
    // -L2 / (scale log2 e) and of -D for its 64 queries.
    for (int i = lane; i < 128 * 2; i += 32) {
      const int r = i >> 1, chunk = i & 1;
      const uint4 v = chunk == 0 ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(ones_smem + C::aug_off(r, chunk * 8)) = v;
    }
    const float inv_sl2 = 1.f / p.scale_log2;
    for (int s = 0; s < n_steps; ++s) {
      const int st = s % C::kStages;
      if (!mbar_wait(&st_full[st], (s / C::kStages) & 1, &abort_flag)) break;
      uint8_t* stat = stages + st * C::kStageBytes + 2 * QT::kBytes;
      const float* nl2 = reinterpret_cast<const float*>(stat + C::kStatLse);
      const float* nd = reinterpret_cast<const float*>(stat + C::kStatD);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = lane + 32 * half;
        __nv_bfloat16 h, m, l;
        split3_bf16(nl2[r] * inv_sl2, h, m, l);
        __nv_bfloat162 hm = __halves2bfloat162(h, m), l0 = __halves2bfloat162(l, __float2bfloat16_rn(0.f));
        *reinterpret_cast<uint4*>(stat + C::kStatAugL + C::aug_off(r, 0)) =
            make_uint4(*reinterpret_cast<uint32_t*>(&hm), *reinterpret_cast<uint32_t*>(&l0), 0u, 0u);
        *reinterpret_cast<uint4*>(stat + C::kStatAugL + C::aug_off(r, 8)) = make_uint4(0u, 0u, 0u, 0u);
        split3_bf16(nd[r], h, m, l);
        hm = __halves2bfloat162(h, m);
        l0 = __halves2bfloat162(l, __float2bfloat16_rn(0.f));
        *reinterpret_cast<uint4*>(stat + C::kStatAugD + C::aug_off(r, 0)) =
            make_uint4(*reinterpret_cast<uint32_t*>(&hm), *reinterpret_cast<uint32_t*>(&l0), 0u, 0u);
        *reinterpret_cast<uint4*>(stat + C::kStatAugD + C::aug_off(r, 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aug_full[st]);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      mbar_arrive_expect_tx(&kv_full, 2 * KV::kBytes);
      for (int c = 0; c < KV::kChunks; ++c) {
        tma_load_4d(&tm_k, &kv_full, k_smem + c * KV::kChunkBytes, c * KV::kRowElems, j, key0, b);
        tma_load_4d(&tm_v, &kv_full, v_smem + c * KV::kChunkBytes, c * KV::kRowElems, j, key0, b);
      }
      int s = 0;
      for (; s < n_steps; ++s) {
        const int st = s % C::kStages;
        if (s >= C::kStages && !mbar_wait(&st_empty[st], ((s / C::kStages) - 1) & 1, &abort_flag)) break;
        const int h = j * p.G + (s_begin + s) / per_head;
        const int q0 = (qs_begin + (s_begin + s) % per_head) * 64;
        uint8_t* dst = stages + st * C::kStageBytes;
        mbar_arrive_expect_tx(&st_full[st], 2 * QT::kBytes + 512);
        for (int c = 0; c < QT::kChunks; ++c) {
          tma_load_4d(&tm_q, &st_full[st], dst + c * QT::kChunkBytes, c * QT::kRowElems, h, q0, b);
          tma_load_4d(&tm_do, &st_full[st], dst + QT::kBytes + c * QT::kChunkBytes, c * QT::kRowElems, h, q0, b);
        }
        const int stat_row = b * p.H_q + h;
        tma_load_2d(&tm_lse2, &st_full[st], dst + 2 * QT::kBytes + C::kStatLse, q0, stat_row);
        tma_load_2d(&tm_dsum, &st_full[st], dst + 2 * QT::kBytes + C::kStatD, q0, stat_row);
      }
      mbar_drain(&kv_full, 0);
      for (int l = max(0, s - C::kStages); l < s; ++l) mbar_drain(&st_full[l % C::kStages], (l / C::kStages) & 1);
    }
  } else if (warp == 1) {
    {
      // ---------------- MMA issuer: whole warp, lane 0 issues ----------------
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // M=128 keys, N=64 queries
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, 0, 1);   // M=128 keys, N=D, B MN-major
      // Descriptors are built once; every MMA only adds a constant offset
      // (a single-thread dependent chain of descriptor arithmetic per MMA
      // would take longer to issue than the MMA takes to run).
      const uint64_t k_kd = KV::kmajor_base(smem_addr(k_smem));
      const uint64_t v_kd = KV::kmajor_base(smem_addr(v_smem));
      const uint64_t st_kd = QT::kmajor_base(smem_addr(stages));
      const uint64_t st_mn = QT::mnmajor_base(smem_addr(stages));
      // Unswizzled K-major: leading (K) byte offset 128, stride (8-row) 256.
      const uint64_t ones_d = smem_desc(smem_addr(ones_smem), 128, 256, kSwNone);
      const uint64_t aug_d = smem_desc(smem_addr(stages + 2 * QT::kBytes + C::kStatAugL), 128, 256, kSwNone);
      auto issue_scores = [&](int s) {
        const int buf = s % C::kBufs;
        const uint64_t q_kd = desc_advance(st_kd, (s % C::kStages) * C::kStageBytes);
        const uint64_t do_kd = desc_advance(q_kd, QT::kBytes);
        // S^T and dP^T accumulate separately: alternating their K steps keeps
        // two independent MMA chains in flight.
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ss_w(tmem + C::col_s(buf), desc_advance(k_kd, KV::kmajor_off(kk)), desc_advance(q_kd, QT::kmajor_off(kk)),
                 idesc_s, kk > 0);
          mma_ss_w(tmem + C::col_dp(buf), desc_advance(v_kd, KV::kmajor_off(kk)),
                 desc_advance(do_kd, QT::kmajor_off(kk)), idesc_s, kk > 0);
        }
        if constexpr (kAug) {  // + (-L2 / (scale log2 e)) and + (-D), per query column
          const uint64_t a0 = desc_advance(aug_d, (s % C::kStages) * C::kStageBytes);
          mma_ss_w(tmem + C::col_s(buf), ones_d, a0, idesc_s, 1u);
          mma_ss_w(tmem + C::col_dp(buf), ones_d, desc_advance(a0, C::kAugBytes), idesc_s, 1u);
        }
        mma_commit_w(&s_full[buf]);
      };
      // A stage's score MMAs need its TMA data and, folded, its statistics.
      // With folded statistics one wait suffices: the statistics warp
      // arrives on aug_full only after it has seen st_full, and that arrive
      // releases what the TMA wrote along with its own stores.
      auto stage_ready = [&](int s) {
        const int st = s % C::kStages;
        const uint32_t ph = (s / C::kStages) & 1;
        if constexpr (kAug) return mbar_wait(&aug_full[st], ph, &abort_flag);
        return mbar_wait(&st_full[st], ph, &abort_flag);
      };
      bool ok = mbar_wait(&kv_full, 0, &abort_flag);
      for (int s = 0; s < C::kBufs && s < n_steps && ok; ++s) {
        ok = stage_ready(s);
        if (ok) {
          tc_fence_after();
          issue_scores(s);
        }
      }
      for (int s = 0; s < n_steps && ok; ++s) {
        const int buf = s % C::kBufs;
        if (!mbar_wait(&p_ready[buf], (s / C::kBufs) & 1, &abort_flag)) break;
        tc_fence_after();
        const uint64_t q_mn = desc_advance(st_mn, (s % C::kStages) * C::kStageBytes);
        const uint64_t do_mn = desc_advance(q_mn, QT::kBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 64 query rows = 4 x K16; dV and dK chains alternate
          mma_ts_w(tmem + C::kColDV, tmem + C::col_s(buf) + kk * 8, desc_advance(do_mn, QT::mnmajor_off(kk)), idesc_g,
                 (s > 0 || kk > 0) ? 1u : 0u);
          mma_ts_w(tmem + C::kColDK, tmem + C::col_dp(buf) + kk * 8, desc_advance(q_mn, QT::mnmajor_off(kk)), idesc_g,
                 (s > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_w(&st_empty[s % C::kStages]);
        if (s + C::kBufs < n_steps) {  // the next scores into the buffer just read
          const int s2 = s + C::kBufs;
          if (!stage_ready(s2)) break;
          tc_fence_after();
          issue_scores(s2);
        }
      }
      mma_commit_w(&mma_done);
    }
  }
  } else {
    regs_alloc<kBwdRegsHigh>();
    // ---------------- softmax-gradient warps ----------------
    const int grp = (warp - 4) >> 2;  // handles steps s with s % 2 == grp
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key row
    const int u = key0 + r;        // key token
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int s = grp; s < n_steps; s += 2) {
      const int buf = s % C::kBufs;
      if (!mbar_wait(&s_full[buf], (s / C::kBufs) & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_col = lane_base + C::col_s(buf), dp_col = lane_base + C::col_dp(buf);
      // Four quarters of 16 query columns, register double-buffered: the
      // next quarter's S^T / dP^T loads are in flight while this one is
      // computed, and each quarter's P^T / dS^T (8 packed words each) go
      // back over columns whose scores have already been read.  Few scores
      // are live at once, which leaves registers for the exponentials of a
      // quarter to overlap.
      uint32_t sa[16], da[16], sb[16], db[16];
      tmem_ld16(s_col, sa);
      tmem_ld16(dp_col, da);
      const uint8_t* stat = stages + (s % C::kStages) * C::kStageBytes + 2 * QT::kBytes;
      const float* l2 = reinterpret_cast<const float*>(stat + C::kStatLse);
      const float* dd = reinterpret_cast<const float*>(stat + C::kStatD);
      const int q0 = (qs_begin + (s_begin + s) % per_head) * 64;
      // Query column c (token q0 + c) contributes iff q0 + c < N and key u
      // is inside its band: u - win_r <= q0 + c <= u + win_l.  Full tiles
      // skip the per-element test.
      int lo = 0, hi = p.N - q0;  // columns [lo, hi) contribute
      if (p.masked) {
        lo = u - p.win_r - q0;
        hi = min(hi, u + p.win_l - q0 + 1);
      }
      const bool full = __all_sync(0xffffffffu, lo <= 0 && hi >= 64);
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      tmem_wait_ld();
      reg_fence16(sa);
      reg_fence16(da);
      // P = 2^(s sl2 - L2), dS = P (dP - D), two columns per packed op; the
      // workspace holds -L2 and -D.  A quarter of the exponentials run as
      // the FMA-pipe polynomial.
      // Folded statistics (kAug): the scores arrive as S^T - L2 / (scale
      // log2 e) and dP^T - D.  Otherwise the quarter's -L2 and -D come as
      // 16-byte shared-memory loads issued one quarter ahead (shared-memory
      // loads of these broadcast values are what kept this loop waiting,
      // hence the folding).
      auto stats = [&](int qt, float4(&lq)[4], float4(&dq4)[4]) {
        if constexpr (!kAug) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            lq[k] = *reinterpret_cast<const float4*>(l2 + qt * 16 + 4 * k);
            dq4[k] = *reinterpret_cast<const float4*>(dd + qt * 16 + 4 * k);
          }
        }
      };
      auto quarter = [&](auto qtc, const uint32_t(&sr)[16], const uint32_t(&dr)[16], const float4(&lq)[4],
                         const float4(&dq4)[4], auto masked) {
        constexpr int qt = decltype(qtc)::value;
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int c2 = 0; c2 < 8; ++c2) {
          const int c = qt * 16 + 2 * c2;  // query column of the pair
          float x0, x1, p0, p1, d0, d1;
          const uint64_t sp = f2_pack(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1]));
          const uint64_t dp = f2_pack(__uint_as_float(dr[2 * c2]), __uint_as_float(dr[2 * c2 + 1]));
          uint64_t t;  // dP - D
          if constexpr (kAug) {
            f2_unpack(f2_mul(sp, sl2x2), x0, x1);
            t = dp;
          } else {
            const float4 l4 = lq[c2 >> 1], d4 = dq4[c2 >> 1];
            const float2 nl = (c2 & 1) ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y);
            const float2 nd = (c2 & 1) ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
            f2_unpack(f2_fma(sp, sl2x2, f2_pack(nl.x, nl.y)), x0, x1);
            t = f2_add(dp, f2_pack(nd.x, nd.y));
          }
          if ((c2 & 3) == 3) {
            exp2_poly_pair(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
          if constexpr (decltype(masked)::value) {
            const bool k0 = c >= lo && c < hi, k1 = c + 1 >= lo && c + 1 < hi;
            p0 = k0 ? p0 : 0.f;
            d0 = k0 ? d0 : 0.f;
            p1 = k1 ? p1 : 0.f;
            d1 = k1 ? d1 : 0.f;
          }
          pk[c2] = pack_bf16x2(p0, p1);
          dk[c2] = pack_bf16x2(d0, d1);
        }
        tmem_st8(s_col + qt * 8, pk);
        tmem_st8(dp_col + qt * 8, dk);
      };
      auto all_quarters = [&](auto masked) {
        float4 la[4], dla[4], lb[4], dlb[4];
        stats(0, la, dla);
        tmem_ld16(s_col + 16, sb);
        tmem_ld16(dp_col + 16, db);
        stats(1, lb, dlb);
        quarter(IntC<0>{}, sa, da, la, dla, masked);
        tmem_wait_ld();
        reg_fence16(sb);
        reg_fence16(db);
        tmem_ld16(s_col + 32, sa);
        tmem_ld16(dp_col + 32, da);
        stats(2, la, dla);
        quarter(IntC<1>{}, sb, db, lb, dlb, masked);
        tmem_wait_ld();
        reg_fence16(sa);
        reg_fence16(da);
        tmem_ld16(s_col + 48, sb);
        tmem_ld16(dp_col + 48, db);
        stats(3, lb, dlb);
        quarter(IntC<2>{}, sa, da, la, dla, masked);
        tmem_wait_ld();
        reg_fence16(sb);
        reg_fence16(db);
        quarter(IntC<3>{}, sb, db, lb, dlb, masked);
      };
      if (full)
        all_quarters(BoolC<false>{});
      else
        all_quarters(BoolC<true>{});
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[buf]);
    }
    // ---------------- epilogue: group 0 writes dV, group 1 writes dK --------
    // With a split, each CTA stages its partial rows over the operand ring
    // (idle once mma_done has fired: every copy into it was consumed by an
    // MMA, and the statistics warp finished before the last one).
    if (ok) ok = mbar_wait(&mma_done, 0, &abort_flag);
    if (ok) {
      tc_fence_after();
      const bool valid = u < p.Nkv;
      const uint32_t col = grp == 0 ? C::kColDV : C::kColDK;
      const float mult = grp == 0 ? 1.f : p.scale;
      GradT* dst = static_cast<GradT*>(grp == 0 ? p.dv : p.dk) +
                   (static_cast<size_t>(b) * p.Nkv + (valid ? u : 0)) * p.ld_dkv + static_cast<size_t>(j) * D;
      float* part = reinterpret_cast<float*>(stages) + (grp * 128 + r) * C::kPartStride;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t rr[16];
        tmem_ld16(lane_base + col + c0, rr);
        tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) v[c] = (n_steps > 0 ? __uint_as_float(rr[c]) : 0.f) * mult;
        if constexpr (kKvSplit) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<float4*>(part + c0)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else if (valid) {
          store16<GradT>(dst + c0, v);
        }
      }
    }
  }

  __syncwarp();
  if constexpr (kKvSplit) {
    // Every CTA of the cluster has staged its partial dV and dK (release /
    // acquire at cluster scope).  CTA `rank` sums rows [r0, r1) of both over
    // the cluster, in rank order, and writes them; the second barrier keeps
    // every CTA's shared memory alive until all reads are done.
    cluster_sync();
    constexpr int kVec = D / 4;  // float4 per row
    const int rows = (128 + splits - 1) / splits;
    const int r0 = rank * rows;
    const int nr = max(0, min(128, r0 + rows) - r0);
    const float* part = reinterpret_cast<const float*>(stages);
    for (int item = threadIdx.x; item < 2 * nr * kVec; item += kBwdThreads) {
      const int which = item / (nr * kVec);  // 0: dV, 1: dK
      const int rem = item - which * nr * kVec;
      const int row = r0 + rem / kVec;
      const int c = (rem % kVec) * 4;
      const float* src = part + (which * 128 + row) * C::kPartStride + c;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < splits; ++q) {
        const float4 w = ld_cluster_f4(map_to_rank(src, static_cast<uint32_t>(q)));
        acc.x += w.x;
        acc.y += w.y;
        acc.z += w.z;
        acc.w += w.w;
      }
      const int tok = key0 + row;
      if (tok < p.Nkv)
        store4<GradT>(static_cast<GradT*>(which == 0 ? p.dv : p.dk) +
                          (static_cast<size_t>(b) * p.Nkv + tok) * p.ld_dkv + static_cast<size_t>(j) * D + c,
                      acc);
    }
    cluster_sync();
  }
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// dQ
// ===========================================================================
template <int D>
struct DqCfg {
  using QT = TileGeo<D, 128>;  // resident Q and dO tiles (packed rows)
  using KS = TileGeo<D, 64>;   // streamed K / V sub-tiles
  static constexpr int kStages = D == 128 ? 4 : 6;
  static constexpr int kStageBytes = 2 * KS::kBytes;
  static constexpr int kSmemBytes = 2 * QT::kBytes + kStages * kStageBytes + 1024;
  static constexpr int kBufs = 3;  // score buffers in TMEM
  // TMEM columns: S/dS and dP of buffer b, then dQ.
  __device__ static constexpr uint32_t col_s(int b) { return 128u * b; }
  __device__ static constexpr uint32_t col_dp(int b) { return 64u + 128u * b; }
  static constexpr uint32_t kColDQ = 128 * kBufs;
  static_assert(kColDQ + D <= 512, "TMEM columns");
  // Split over a cluster: partial dQ rows staged over the ring.
  static constexpr int kPartStride = D + 4;  // floats per row; the pad spreads rows over the banks
  static_assert(128 * kPartStride * 4 <= kStages * kStageBytes, "partial dQ fits over the ring");
};

// kKvSplit: the instantiation launched in clusters that split each query
// tile's key sub-tiles (p.kv_splits > 1, unmasked problems only); the other
// one carries none of that code.
template <int D, typename GradT, bool kKvSplit = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p) {
  using C = DqCfg<D>;
  using QT = typename C::QT;
  using KS = typename C::KS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t st_full[C::kStages];
  __shared__ __align__(8) uint64_t st_empty[C::kStages];
  __shared__ __align__(8) uint64_t s_full[C::kBufs];
  __shared__ __align__(8) uint64_t p_ready[C::kBufs];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* do_smem = smem + QT::kBytes;
  uint8_t* stages = smem + 2 * QT::kBytes;

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const int T = 128 >> p.log2g;
  const BlockUnit u = block_unit(p.longest_first);
  const int ux = kKvSplit ? u.x / p.kv_splits : u.x;
  const int tblk = p.longest_first ? (p.n_tblk - 1 - ux) : ux;
  const int j = u.y / p.n_sub;
  const int sub = u.y % p.n_sub;
  const int b = u.z;
  const int h0 = j * p.G + sub * p.g;
  const int t0 = tblk * T;
  const int last_tok = min(t0 + T, p.N) - 1;
  // Keys visible to some row of the tile: [t0 - win_l, last_tok + win_r]
  // within [0, Nkv), streamed as 64-key sub-tiles from ks_begin.
  const int k_lo = p.masked ? max(0, t0 - p.win_l) : 0;
  const int k_hi = p.masked ? min(p.Nkv, last_tok + p.win_r + 1) : p.Nkv;
  int ks_begin = k_lo / 64;
  int n_steps = max(0, (k_hi + 63) / 64 - ks_begin);
  // Few query tiles against many keys: the key sub-tiles are split over a
  // cluster of p.kv_splits CTAs (CTA `rank` takes a contiguous share) and the
  // partial dQ rows summed through distributed shared memory at the end.
  const int splits = kKvSplit ? p.kv_splits : 1;
  const int rank = kKvSplit ? static_cast<int>(cluster_rank()) : 0;
  if constexpr (kKvSplit) {
    const int a0 = static_cast<int>(static_cast<long long>(n_steps) * rank / splits);
    const int a1 = static_cast<int>(static_cast<long long>(n_steps) * (rank + 1) / splits);
    ks_begin += a0;
    n_steps = a1 - a0;
  }

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    for (int t = 0; t < C::kBufs; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_ready[t], 4);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  // Programmatic dependent launch: the set-up above may overlap the end of
  // the previous kernel on the stream; nothing below touches global memory
  // before that kernel has completed.  Dependents are released only after
  // the barrier, once this CTA holds its TMEM: a dependent CTA that took the
  // SM's columns first would wait for this grid while this CTA waited for
  // the columns.
  // Launched right after dK/dV (wait_at_exit), this grid reads nothing that
  // grid writes: the inputs and the preprocess's statistics are complete
  // once it may start (every dK/dV CTA releases its dependents only after
  // its own wait on the preprocess has returned), so the work need not wait
  // for dK/dV.  The wait moves to the exit, so that a kernel after this one
  // on the stream still finds dK/dV complete.
  if (!p.wait_at_exit) grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = tmem_base_sh;

  if (warp < 4) {
  regs_dealloc<kBwdRegsLow>();
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, 2 * QT::kBytes);
      for (int c = 0; c < QT::kChunks; ++c) {
        tma_load_4d(&tm_q, &q_full, q_smem + c * QT::kChunkBytes, c * QT::kRowElems, h0, t0, b);
        tma_load_4d(&tm_do, &q_full, do_smem + c * QT::kChunkBytes, c * QT::kRowElems, h0, t0, b);
      }
      int s = 0;
      for (; s < n_steps; ++s) {
        const int st = s % C::kStages;
        if (s >= C::kStages && !mbar_wait(&st_empty[st], ((s / C::kStages) - 1) & 1, &abort_flag)) break;
        uint8_t* dst = stages + st * C::kStageBytes;
        mbar_arrive_expect_tx(&st_full[st], 2 * KS::kBytes);
        for (int c = 0; c < KS::kChunks; ++c) {
          const int key = (ks_begin + s) * 64;
          tma_load_4d(&tm_k, &st_full[st], dst + c * KS::kChunkBytes, c * KS::kRowElems, j, key, b);
          tma_load_4d(&tm_v, &st_full[st], dst + KS::kBytes + c * KS::kChunkBytes, c * KS::kRowElems, j, key, b);
        }
      }
      mbar_drain(&q_full, 0);
      for (int l = max(0, s - C::kStages); l < s; ++l) mbar_drain(&st_full[l % C::kStages], (l / C::kStages) & 1);
    }
  } else if (warp == 1) {
    {  // MMA issuer: whole warp, lane 0 issues
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // M=128 rows, N=64 keys
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, 0, 1);   // M=128 rows, N=D, B MN-major
      // Descriptors built once; each MMA adds a constant offset.
      const uint64_t q_kd = QT::kmajor_base(smem_addr(q_smem));
      const uint64_t do_kd = QT::kmajor_base(smem_addr(do_smem));
      const uint64_t st_kd = KS::kmajor_base(smem_addr(stages));
      const uint64_t st_mn = KS::mnmajor_base(smem_addr(stages));
      auto issue_scores = [&](int s) {
        const int buf = s % C::kBufs;
        const uint64_t k_kd = desc_advance(st_kd, (s % C::kStages) * C::kStageBytes);
        const uint64_t v_kd = desc_advance(k_kd, KS::kBytes);
        // S and dP accumulate separately: alternate their K steps.
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ss_w(tmem + C::col_s(buf), desc_advance(q_kd, QT::kmajor_off(kk)), desc_advance(k_kd, KS::kmajor_off(kk)),
                 idesc_s, kk > 0);
          mma_ss_w(tmem + C::col_dp(buf), desc_advance(do_kd, QT::kmajor_off(kk)),
                 desc_advance(v_kd, KS::kmajor_off(kk)), idesc_s, kk > 0);
        }
        mma_commit_w(&s_full[buf]);
      };
      bool ok = mbar_wait(&q_full, 0, &abort_flag);
      for (int s = 0; s < C::kBufs && s < n_steps && ok; ++s) {
        ok = mbar_wait(&st_full[s % C::kStages], (s / C::kStages) & 1, &abort_flag);
        if (ok) {
          tc_fence_after();
          issue_scores(s);
        }
      }
      for (int s = 0; s < n_steps && ok; ++s) {
        const int buf = s % C::kBufs;
        if (!mbar_wait(&p_ready[buf], (s / C::kBufs) & 1, &abort_flag)) break;
        tc_fence_after();
        const uint64_t k_mn = desc_advance(st_mn, (s % C::kStages) * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 64 keys = 4 x K16
          mma_ts_w(tmem + C::kColDQ, tmem + C::col_s(buf) + kk * 8, desc_advance(k_mn, KS::mnmajor_off(kk)), idesc_g,
                 (s > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(&st_empty[s % C::kStages]);
        if (s + C::kBufs < n_steps) {  // the next scores into the buffer just read
          const int s2 = s + C::kBufs;
          if (!mbar_wait(&st_full[s2 % C::kStages], (s2 / C::kStages) & 1, &abort_flag)) break;
          tc_fence_after();
          issue_scores(s2);
        }
      }
      mma_commit_w(&mma_done);
    }
  }
  } else {
    regs_alloc<kBwdRegsHigh>();
    const int grp = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int tok = t0 + (r >> p.log2g);
    const int head = h0 + (r & (p.g - 1));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    const size_t stat = (static_cast<size_t>(b) * p.H_q + head) * p.n_pad + tok;  // tok < n_pad
    const float nl2 = p.lse2[stat];  // -LSE * log2(e)
    const float ndd = p.dsum[stat];  // -D
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t nl2x2 = f2_pack(nl2, nl2);
    const uint64_t ndd2 = f2_pack(ndd, ndd);
    bool ok = true;
    for (int s = grp; s < n_steps; s += 2) {
      const int buf = s % C::kBufs;
      if (!mbar_wait(&s_full[buf], (s / C::kBufs) & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_col = lane_base + C::col_s(buf), dp_col = lane_base + C::col_dp(buf);
      // Four register double-buffered quarters of 16 keys, as in the dK/dV
      // kernel: loads of the next quarter overlap this one's arithmetic and
      // each quarter's dS (8 packed words) goes back over scores already read.
      uint32_t sa[16], da[16], sb[16], db[16];
      tmem_ld16(s_col, sa);
      tmem_ld16(dp_col, da);
      const int kbase = (ks_begin + s) * 64;
      int lo = 0, hi = p.Nkv - kbase;  // keys [lo, hi) of the sub-tile are visible
      if (p.masked) {
        lo = tok - p.win_l - kbase;
        hi = min(hi, tok + p.win_r - kbase + 1);
      }
      const bool full = __all_sync(0xffffffffu, lo <= 0 && hi >= 64);
      tmem_wait_ld();
      reg_fence16(sa);
      reg_fence16(da);
      // dS = 2^(s sl2 - L2) (dP - D) with the row's -L2 and -D (nl2, ndd),
      // two keys per packed op, a quarter of the exponentials as the
      // FMA-pipe polynomial; full tiles skip the per-element key test.
      auto quarter = [&](auto qtc, const uint32_t(&sr)[16], const uint32_t(&dr)[16], auto masked) {
        constexpr int qt = decltype(qtc)::value;
        uint32_t dk[8];
#pragma unroll
        for (int c2 = 0; c2 < 8; ++c2) {
          const int c = qt * 16 + 2 * c2;  // key column of the pair
          float x0, x1, p0, p1, d0, d1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1])), sl2x2, nl2x2), x0,
                    x1);
          if ((c2 & 3) == 3) {
            exp2_poly_pair(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          const uint64_t t = f2_add(f2_pack(__uint_as_float(dr[2 * c2]), __uint_as_float(dr[2 * c2 + 1])), ndd2);
          f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
          if constexpr (decltype(masked)::value) {
            d0 = (c >= lo && c < hi) ? d0 : 0.f;
            d1 = (c + 1 >= lo && c + 1 < hi) ? d1 : 0.f;
          }
          dk[c2] = pack_bf16x2(d0, d1);
        }
        tmem_st8(s_col + qt * 8, dk);
      };
      auto all_quarters = [&](auto masked) {
        tmem_ld16(s_col + 16, sb);
        tmem_ld16(dp_col + 16, db);
        quarter(IntC<0>{}, sa, da, masked);
        tmem_wait_ld();
        reg_fence16(sb);
        reg_fence16(db);
        tmem_ld16(s_col + 32, sa);
        tmem_ld16(dp_col + 32, da);
        quarter(IntC<1>{}, sb, db, masked);
        tmem_wait_ld();
        reg_fence16(sa);
        reg_fence16(da);
        tmem_ld16(s_col + 48, sb);
        tmem_ld16(dp_col + 48, db);
        quarter(IntC<2>{}, sa, da, masked);
        tmem_wait_ld();
        reg_fence16(sb);
        reg_fence16(db);
        quarter(IntC<3>{}, sb, db, masked);
      };
      if (full)
        all_quarters(BoolC<false>{});
      else
        all_quarters(BoolC<true>{});
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[buf]);
    }
    if (ok) ok = mbar_wait(&mma_done, 0, &abort_flag);
    if (ok) {
      tc_fence_after();
      const bool valid = tok < p.N;
      GradT* dst = static_cast<GradT*>(p.dq) + (static_cast<size_t>(b) * p.N + (valid ? tok : 0)) * p.ld_dq +
                   static_cast<size_t>(head) * D;
      // With a split, the partial row is staged over the operand ring (idle
      // once mma_done has fired: every copy into it was consumed by an MMA).
      float* part = reinterpret_cast<float*>(stages) + r * C::kPartStride;
      // The two groups split the columns of dQ (group 0 alone when D = 16).
      constexpr int kHalf = D >= 32 ? D / 2 : D;
#pragma unroll 1
      for (int c0 = grp * kHalf; c0 < (grp + 1) * kHalf && c0 < D; c0 += 16) {
        uint32_t rr[16];
        tmem_ld16(lane_base + C::kColDQ + c0, rr);
        tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) v[c] = (n_steps > 0 ? __uint_as_float(rr[c]) : 0.f) * p.scale;
        if constexpr (kKvSplit) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<float4*>(part + c0)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else if (valid) {
          store16<GradT>(dst + c0, v);
        }
      }
    }
  }

  __syncwarp();
  if constexpr (kKvSplit) {
    // Every CTA of the cluster has staged its partial dQ rows (release /
    // acquire at cluster scope).  CTA `rank` sums rows [r0, r0 + nr) over the
    // cluster, in rank order, and writes them; the second barrier keeps every
    // CTA's shared memory alive until all reads are done.
    cluster_sync();
    constexpr int kVec = D / 4;  // float4 per row
    const int rows = (128 + splits - 1) / splits;
    const int r0 = rank * rows;
    const int nr = max(0, min(128, r0 + rows) - r0);
    const float* part = reinterpret_cast<const float*>(stages);
    for (int item = threadIdx.x; item < nr * kVec; item += kBwdThreads) {
      const int row = r0 + item / kVec;
      const int c = (item % kVec) * 4;
      const int tok_r = t0 + (row >> p.log2g);
      if (tok_r >= p.N) continue;
      const float* src = part + row * C::kPartStride + c;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < splits; ++q) {
        const float4 w = ld_cluster_f4(map_to_rank(src, static_cast<uint32_t>(q)));
        acc.x += w.x;
        acc.y += w.y;
        acc.z += w.z;
        acc.w += w.w;
      }
      store4<GradT>(static_cast<GradT*>(p.dq) + (static_cast<size_t>(b) * p.N + tok_r) * p.ld_dq +
                        static_cast<size_t>(h0 + (row & (p.g - 1))) * D + c,
                    acc);
    }
    cluster_sync();
  }
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (p.wait_at_exit) grid_dependency_wait();
}

}  // namespace sqa
