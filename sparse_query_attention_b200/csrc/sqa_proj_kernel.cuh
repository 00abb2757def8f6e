// sqa_proj_kernel.cuh - the projection GEMMs of an SQA layer on the sm_100a
// tensor cores:  C[M, N] (+)= sum_k A(m, k) B(n, k) (+ bias[n]).
//
// In Sparse Query Attention the query projection produces only H_q * d_head
// columns and the output projection consumes only H_q * d_head ("ReactiveAI/
// xSMQAT-m" model card, note on model size); the key/value projections keep
// H_kv * d_head.  The forward of all four is C = X W^T; their backward is
// dX = dY W and dW = dY^T X.  The operands are therefore taken as stored,
// either K-contiguous (A[m][k], B[n][k]: activations, nn.Linear weights) or
// MN-contiguous (A[k][m], B[k][n]), and read with the matching shared-memory
// operand layout, so no transpose ever goes through memory.
//
// Design: a persistent kernel, one CTA per SM walking the 128 x BN output
// tiles in groups of row tiles (all column tiles of a group before the next;
// the group size is chosen so that the CTAs running together find their A
// and B tiles in L2 and each operand comes from DRAM about once), eight warps:
//   warp 0 / one lane : TMA producer, 64-wide K slices of A and B into a
//                       4-stage ring (128-byte swizzle) that runs on across
//                       tiles.
//   warp 1            : issues tcgen05.mma (M=128, N=BN, K=16) from
//                       warp-uniform code (lane 0 issues) into one of two
//                       TMEM accumulators, alternating per tile, and commits
//                       each stage back to the producer.
//   warp 2            : TMEM allocation.
//   warps 4-7         : epilogue of the previous tile, TMEM -> registers
//                       (+C, +bias) -> global, while the next tile's
//                       mainloop runs into the other accumulator.
#pragma once

#include "sqa_ptx.cuh"

namespace sqa {

constexpr int kProjBM = 128;
constexpr int kProjBK = 64;
constexpr int kProjStages = 4;

template <int BN>
struct ProjSmem {
  static constexpr int kABytes = kProjBM * kProjBK * 2;
  static constexpr int kBBytes = BN * kProjBK * 2;
  static constexpr int kTileBytes = kProjStages * (kABytes + kBBytes);
  static constexpr int kDynamicBytes = kTileBytes + 1024;  // + alignment slack
};

// kAMN / kBMN: operand stored MN-contiguous (A[k][m] / B[k][n]) instead of
// K-contiguous (A[m][k] / B[n][k]).  An MN-contiguous tile is loaded as
// 64 (MN) x 64 (K) boxes, one 8 KB chunk per 64 rows of M or N.
constexpr int kProjThreads = 256;

// Output tile of linear index `tile`: groups of `group_m` row tiles, all
// column tiles of a group before the next group, rows fastest inside it.
// group_m = 1 walks N fastest (every B tile stays hot in L2 while A streams
// through once); group_m >= m_tiles walks M fastest (A stays, B streams once).
// The host picks the raster from the operand sizes.
__device__ __forceinline__ void proj_tile_coords(int tile, int m_tiles, int n_tiles, int group_m, int& mt,
                                                 int& nt) {
  const int per_group = group_m * n_tiles;
  const int group = tile / per_group;
  const int first = group * group_m;
  const int gm = min(group_m, m_tiles - first);
  const int local = tile - group * per_group;
  mt = first + local % gm;
  nt = local / gm;
}

template <int BN, bool kOutBf16, bool kAMN, bool kBMN>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const float* __restrict__ bias, void* __restrict__ y, int M, int K, int Nout, int accumulate,
                     int group_m) {
  static_assert(!kBMN || BN % 64 == 0, "MN-contiguous B needs BN in 64, 128, 256");
  using S = ProjSmem<BN>;
  constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;  // one accumulator
  constexpr uint32_t kTmemCols = 2 * kAccCols;        // two, alternating per tile
  constexpr uint32_t kMnChunk = 64 * 128;             // one 64 x 64 MN-contiguous box
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kProjStages];
  __shared__ __align__(8) uint64_t empty_bar[kProjStages];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + kProjStages * S::kABytes;

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + kProjBM - 1) / kProjBM;
  const int n_tiles = (Nout + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (K + kProjBK - 1) / kProjBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kProjStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);  // the four epilogue warps
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
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
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer; g counts k-blocks over all of this CTA's tiles.
      int g = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        proj_tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
        const int m0 = mt * kProjBM;
        const int n0 = nt * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % kProjStages;
          const uint32_t ph = (g / kProjStages) & 1;
          if (g >= kProjStages && !mbar_wait(&empty_bar[s], ph ^ 1, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[s], S::kABytes + S::kBBytes);
          uint8_t* a_dst = a_tiles + s * S::kABytes;
          uint8_t* b_dst = b_tiles + s * S::kBBytes;
          if constexpr (kAMN) {
            for (int c = 0; c < kProjBM / 64; ++c)
              tma_load_2d(&tm_a, &full_bar[s], a_dst + c * kMnChunk, m0 + 64 * c, kb * kProjBK);
          } else {
            tma_load_2d(&tm_a, &full_bar[s], a_dst, kb * kProjBK, m0);
          }
          if constexpr (kBMN) {
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(&tm_b, &full_bar[s], b_dst + c * kMnChunk, n0 + 64 * c, kb * kProjBK);
          } else {
            tma_load_2d(&tm_b, &full_bar[s], b_dst, kb * kProjBK, n0);
          }
        }
      }
      // No copy may still be landing in shared memory when the CTA exits.
      for (int q = g > kProjStages ? g - kProjStages : 0; q < g; ++q)
        mbar_drain(&full_bar[q % kProjStages], (q / kProjStages) & 1);
    }
  } else if (warp == 1) {
    // MMA issuer: the whole warp runs the loop (operands stay warp-uniform),
    // lane 0 issues.  Descriptors are built once and advanced by offsets:
    // a K-contiguous operand steps 32 bytes along its 128-byte rows per
    // 16-wide K step; an MN-contiguous one steps 16 rows of 128 bytes, with
    // its 64-wide MN chunks kMnChunk bytes apart.
    constexpr uint32_t idesc = idesc_bf16_f32(kProjBM, BN, kAMN ? 1 : 0, kBMN ? 1 : 0);
    const uint64_t a_desc0 = kAMN ? smem_desc(smem_addr(a_tiles), kMnChunk, 1024, kSw128)
                                  : smem_desc(smem_addr(a_tiles), 16, 1024, kSw128);
    const uint64_t b_desc0 = kBMN ? smem_desc(smem_addr(b_tiles), kMnChunk, 1024, kSw128)
                                  : smem_desc(smem_addr(b_tiles), 16, 1024, kSw128);
    constexpr uint32_t kAStep = kAMN ? 16 * 128 : 32;
    constexpr uint32_t kBStep = kBMN ? 16 * 128 : 32;
    int g = 0;
    bool ok = true;
    for (int tile = blockIdx.x, k = 0; tile < num_tiles && ok; tile += gridDim.x, ++k) {
      const int acc = k & 1;
      // The epilogue has read this accumulator's previous tile.
      if (k >= 2 && !mbar_wait(&acc_empty[acc], ((k >> 1) - 1) & 1, &abort_flag)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + acc * kAccCols;
      for (int kb = 0; kb < num_kb; ++kb, ++g) {
        const int s = g % kProjStages;
        const uint32_t ph = (g / kProjStages) & 1;
        if (!mbar_wait(&full_bar[s], ph, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = desc_advance(a_desc0, s * S::kABytes);
        const uint64_t bd = desc_advance(b_desc0, s * S::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kProjBK / 16; ++kk)
          mma_ss_w(tacc, desc_advance(ad, kk * kAStep), desc_advance(bd, kk * kBStep), idesc, (kb | kk) != 0);
        mma_commit_w(&empty_bar[s]);
      }
      if (ok) mma_commit_w(&acc_full[acc]);
    }
    mma_commit_w(&mma_done);
  } else if (warp >= 4) {
    // Epilogue: warp w reads TMEM lanes [32 (w - 4), +32) = output rows.
    const int wq = warp & 3;
    for (int tile = blockIdx.x, k = 0; tile < num_tiles; tile += gridDim.x, ++k) {
      const int acc = k & 1;
      if (!mbar_wait(&acc_full[acc], (k >> 1) & 1, &abort_flag)) break;
      tc_fence_after();
      int mt, nt;
      proj_tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
      const int row = mt * kProjBM + wq * 32 + lane;
      const int n0 = nt * BN;
      const uint32_t lane_addr = tmem + acc * kAccCols + (static_cast<uint32_t>(wq * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(lane_addr + c0, r);
        tmem_wait_ld();
        const int n = n0 + c0;
        if (row < M && n < Nout) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]) + (bias != nullptr ? bias[n + i] : 0.f);
          if constexpr (kOutBf16) {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(row) * Nout + n);
            dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
            dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + static_cast<size_t>(row) * Nout + n);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 w = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
              if (accumulate) {
                const float4 old = dst[i];
                w.x += old.x;
                w.y += old.y;
                w.z += old.z;
                w.w += old.w;
              }
              dst[i] = w;
            }
          }
        }
      }
      // Hand the accumulator back to the MMA warp.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  // ---- teardown: every MMA the issuer started has finished -----------------
  __syncwarp();
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ===========================================================================
// The same GEMM over CTA pairs, for K-contiguous A and B (activations times
// nn.Linear weights, the layer's forward projections): 256 x 256 output
// tiles, one per pair.  Each CTA loads its own 128 rows of A and 128 of the
// 256 rows of B (output columns) per 64-wide K slice, 32 KB instead of the
// 48 KB a single CTA needs for a 128 x 256 tile, so six stages fit and the
// ring covers ~1.5x the L2 latency of the single-CTA kernel.  The even CTA's
// MMA warp issues one tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) per
// K step; both CTAs' copies complete on the even CTA's "full" barrier, the
// even CTA's commits arrive on both CTAs' "empty" and accumulator barriers,
// and both CTAs' epilogue warps arrive on the even CTA's accumulator-free
// barrier.  Each CTA's epilogue writes its own 128 rows from its own TMEM.
// ===========================================================================
constexpr int kPairBN = 256;  // output columns per pair tile (128 per CTA's B half)
constexpr int kPairStages = 6;
constexpr int kPairHalfBytes = kProjBM * kProjBK * 2;  // 16 KB: A rows or B rows of one CTA, one K slice
constexpr int kPairDynamicBytes = kPairStages * 2 * kPairHalfBytes + 1024;

template <bool kOutBf16>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const float* __restrict__ bias, void* __restrict__ y, int M, int K, int Nout,
                          int accumulate, int group_m) {
  constexpr uint32_t kAccCols = kPairBN;       // one accumulator: 128 lanes x 256 columns per CTA
  constexpr uint32_t kTmemCols = 2 * kAccCols;  // two, alternating per tile
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPairStages];   // used in the even CTA
  __shared__ __align__(8) uint64_t empty_bar[kPairStages];  // both
  __shared__ __align__(8) uint64_t acc_full[2];             // both
  __shared__ __align__(8) uint64_t acc_empty[2];            // used in the even CTA
  __shared__ __align__(8) uint64_t mma_done;                // both
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + kPairStages * kPairHalfBytes;

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_tiles = (M + 2 * kProjBM - 1) / (2 * kProjBM);
  const int n_tiles = (Nout + kPairBN - 1) / kPairBN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (K + kProjBK - 1) / kProjBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // four epilogue warps in each CTA
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(&tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  // Programmatic dependent launch as in proj_gemm_kernel; the cluster
  // barrier makes both CTAs' barrier initialisation and TMEM allocation
  // visible to the pair before either uses the other's.
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer of this CTA; g counts k-blocks over the pair's tiles.
      const uint32_t full0 = map_to_rank(&full_bar[0], 0);  // the even CTA's full barriers
      int g = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
        int mt, nt;
        proj_tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
        const int m0 = mt * 2 * kProjBM + static_cast<int>(rank) * kProjBM;
        const int n0 = nt * kPairBN + static_cast<int>(rank) * kProjBM;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % kPairStages;
          const uint32_t ph = (g / kPairStages) & 1;
          if (g >= kPairStages && !mbar_wait(&empty_bar[s], ph ^ 1, &abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 4 * kPairHalfBytes);  // both CTAs' A and B
          const uint32_t fb = full0 + s * static_cast<uint32_t>(sizeof(uint64_t));
          tma_load_2d_pair(&tm_a, fb, a_tiles + s * kPairHalfBytes, kb * kProjBK, m0);
          tma_load_2d_pair(&tm_b, fb, b_tiles + s * kPairHalfBytes, kb * kProjBK, n0);
        }
      }
      // No copy of this CTA may still be landing in its shared memory when
      // it exits: the even CTA drains its full barriers (which count both
      // CTAs' copies); the odd CTA's last copies are covered by the MMAs
      // that consumed them (mma_done) or, after an abort, by the final
      // cluster barrier following the even CTA's drain.
      if (rank == 0)
        for (int q = g > kPairStages ? g - kPairStages : 0; q < g; ++q)
          mbar_drain(&full_bar[q % kPairStages], (q / kPairStages) & 1);
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // MMA issuer of the pair: the whole warp runs the loop, one lane issues.
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kProjBM, kPairBN, 0, 0);
      const uint64_t a_desc0 = smem_desc(smem_addr(a_tiles), 16, 1024, kSw128);
      const uint64_t b_desc0 = smem_desc(smem_addr(b_tiles), 16, 1024, kSw128);
      int g = 0;
      bool ok = true;
      for (int tile = pair, k = 0; tile < num_tiles && ok; tile += n_pairs, ++k) {
        const int acc = k & 1;
        // Both CTAs' epilogues have read this accumulator's previous tile.
        if (k >= 2 && !mbar_wait(&acc_empty[acc], ((k >> 1) - 1) & 1, &abort_flag)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + acc * kAccCols;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % kPairStages;
          const uint32_t ph = (g / kPairStages) & 1;
          if (!mbar_wait(&full_bar[s], ph, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc_advance(a_desc0, s * kPairHalfBytes);
          const uint64_t bd = desc_advance(b_desc0, s * kPairHalfBytes);
#pragma unroll
          for (int kk = 0; kk < kProjBK / 16; ++kk)
            mma_ss_pair_w(tacc, desc_advance(ad, kk * 32), desc_advance(bd, kk * 32), idesc, (kb | kk) != 0);
          mma_commit_pair_w(&empty_bar[s]);
        }
        if (ok) mma_commit_pair_w(&acc_full[acc]);
      }
      mma_commit_pair_w(&mma_done);
    }
  } else if (warp >= 4) {
    // Epilogue: warp w reads TMEM lanes [32 (w - 4), +32) = this CTA's output rows.
    const int wq = warp & 3;
    const uint32_t acc_empty0 = map_to_rank(&acc_empty[0], 0);
    for (int tile = pair, k = 0; tile < num_tiles; tile += n_pairs, ++k) {
      const int acc = k & 1;
      if (!mbar_wait(&acc_full[acc], (k >> 1) & 1, &abort_flag)) break;
      tc_fence_after();
      int mt, nt;
      proj_tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
      const int row = mt * 2 * kProjBM + static_cast<int>(rank) * kProjBM + wq * 32 + lane;
      const int n0 = nt * kPairBN;
      const uint32_t lane_addr = tmem + acc * kAccCols + (static_cast<uint32_t>(wq * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < kPairBN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(lane_addr + c0, r);
        tmem_wait_ld();
        const int n = n0 + c0;
        if (row < M && n < Nout) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]) + (bias != nullptr ? bias[n + i] : 0.f);
          if constexpr (kOutBf16) {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(row) * Nout + n);
            dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
            dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + static_cast<size_t>(row) * Nout + n);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 w = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
              if (accumulate) {
                const float4 old = dst[i];
                w.x += old.x;
                w.y += old.y;
                w.z += old.z;
                w.w += old.w;
              }
              dst[i] = w;
            }
          }
        }
      }
      // Hand the accumulator back to the even CTA's MMA warp.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty0 + acc * static_cast<uint32_t>(sizeof(uint64_t)));
    }
  }

  // ---- teardown: every MMA of the pair has finished, in both CTAs ----------
  __syncwarp();
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still arrive on its barriers
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ===========================================================================
// Split K over a thread-block cluster, for products with few output tiles and
// a long K: the weight gradients of a layer, dW = dY^T X, contract over all
// B * N tokens into a d_model-sized tile grid that would otherwise leave all
// but a few SMs idle.  Each cluster of S CTAs (S in 2, 4, 8) computes one
// 128 x BN output tile; CTA r of the cluster contracts K blocks
// [r num_kb / S, (r + 1) num_kb / S) into its TMEM accumulator.  Once its
// last MMA has finished, each CTA stages its fp32 partial tile in its own
// shared memory (over the operand ring, idle by then), and after a cluster
// barrier CTA r sums rows [r 128 / S, (r + 1) 128 / S) of all S partials
// through distributed shared memory, in rank order, and writes them (bias,
// accumulate and output type as in proj_gemm_kernel).  The sum order is
// fixed, so results are the same from run to run; no workspace is needed.
// Warp roles as in proj_gemm_kernel, one tile per cluster; the ring is as
// deep as ~192 KB of shared memory allows (up to 8 stages), since each CTA's
// share of K is short and latency, not the tensor pipe, bounds it.
// ===========================================================================
template <int BN>
struct SplitSmem {
  static constexpr int kABytes = kProjBM * kProjBK * 2;
  static constexpr int kBBytes = BN * kProjBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024 / kStageBytes) < 8 ? (192 * 1024 / kStageBytes) : 8;
  static constexpr int kPartStride = BN + 4;  // floats per staged row; the pad spreads rows over the banks
  static_assert(kProjBM * kPartStride * 4 <= kStages * kStageBytes, "the partial tile fits over the ring");
  static constexpr int kDynamicBytes = kStages * kStageBytes + 1024;
};

template <int BN, bool kOutBf16, bool kAMN, bool kBMN>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                            const float* __restrict__ bias, void* __restrict__ y, int M, int K, int Nout,
                            int accumulate) {
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 64, "split-K tiles are 128 x 32 or 128 x 64");
  static_assert(!kBMN || BN == 64, "MN-contiguous B is loaded as 64-column boxes");
  using S = SplitSmem<BN>;
  constexpr int kStages = S::kStages;
  constexpr uint32_t kTmemCols = BN;  // one accumulator
  constexpr uint32_t kMnChunk = 64 * 128;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + kStages * S::kABytes;
  float* part = reinterpret_cast<float*>(smem);  // [128][kPartStride], once the ring is idle

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const int splits = static_cast<int>(cluster_num_ctas());
  const int rank = static_cast<int>(cluster_rank());
  const int n_tiles = (Nout + BN - 1) / BN;
  const int tile = static_cast<int>(blockIdx.x) / splits;
  const int m0 = (tile / n_tiles) * kProjBM;
  const int n0 = (tile % n_tiles) * BN;
  const int num_kb = (K + kProjBK - 1) / kProjBK;
  const int kb0 = static_cast<int>(static_cast<long long>(num_kb) * rank / splits);
  const int kb1 = static_cast<int>(static_cast<long long>(num_kb) * (rank + 1) / splits);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  // Programmatic dependent launch as in proj_gemm_kernel.
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer over this CTA's K blocks.
      int g = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int s = g % kStages;
        if (g >= kStages && !mbar_wait(&empty_bar[s], ((g / kStages) & 1) ^ 1, &abort_flag)) break;
        mbar_arrive_expect_tx(&full_bar[s], S::kABytes + S::kBBytes);
        uint8_t* a_dst = a_tiles + s * S::kABytes;
        uint8_t* b_dst = b_tiles + s * S::kBBytes;
        if constexpr (kAMN) {
          for (int c = 0; c < kProjBM / 64; ++c)
            tma_load_2d(&tm_a, &full_bar[s], a_dst + c * kMnChunk, m0 + 64 * c, kb * kProjBK);
        } else {
          tma_load_2d(&tm_a, &full_bar[s], a_dst, kb * kProjBK, m0);
        }
        if constexpr (kBMN) {
          tma_load_2d(&tm_b, &full_bar[s], b_dst, n0, kb * kProjBK);
        } else {
          tma_load_2d(&tm_b, &full_bar[s], b_dst, kb * kProjBK, n0);
        }
      }
      // No copy may still be landing in shared memory once the ring is reused.
      for (int q = g > kStages ? g - kStages : 0; q < g; ++q) mbar_drain(&full_bar[q % kStages], (q / kStages) & 1);
    }
  } else if (warp == 1) {
    // MMA issuer (whole warp in the loop, lane 0 issues), as in proj_gemm_kernel.
    constexpr uint32_t idesc = idesc_bf16_f32(kProjBM, BN, kAMN ? 1 : 0, kBMN ? 1 : 0);
    const uint64_t a_desc0 = kAMN ? smem_desc(smem_addr(a_tiles), kMnChunk, 1024, kSw128)
                                  : smem_desc(smem_addr(a_tiles), 16, 1024, kSw128);
    const uint64_t b_desc0 = kBMN ? smem_desc(smem_addr(b_tiles), kMnChunk, 1024, kSw128)
                                  : smem_desc(smem_addr(b_tiles), 16, 1024, kSw128);
    constexpr uint32_t kAStep = kAMN ? 16 * 128 : 32;
    constexpr uint32_t kBStep = kBMN ? 16 * 128 : 32;
    bool ok = true;
    int g = 0;
    for (int kb = kb0; kb < kb1; ++kb, ++g) {
      const int s = g % kStages;
      if (!mbar_wait(&full_bar[s], (g / kStages) & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t ad = desc_advance(a_desc0, s * S::kABytes);
      const uint64_t bd = desc_advance(b_desc0, s * S::kBBytes);
#pragma unroll
      for (int kk = 0; kk < kProjBK / 16; ++kk)
        mma_ss_w(tmem, desc_advance(ad, kk * kAStep), desc_advance(bd, kk * kBStep), idesc, (g | kk) != 0);
      mma_commit_w(&empty_bar[s]);
    }
    if (ok) mma_commit_w(&acc_full);
    mma_commit_w(&mma_done);
  } else if (warp >= 4) {
    // Stage this CTA's partial tile: TMEM lane (row) -> its padded smem row.
    // acc_full fires after the last MMA has finished reading the ring, and
    // every copy into the ring was waited for before its MMA was issued.
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    if (mbar_wait(&acc_full, 0, &abort_flag)) {
      tc_fence_after();
      float* dst = part + row * S::kPartStride;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(lane_addr + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(dst + c0)[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                               __uint_as_float(r[4 * i + 2]),
                                                               __uint_as_float(r[4 * i + 3]));
      }
    }
  }
  __syncwarp();
  // Every CTA's partial is staged (release / acquire at cluster scope).
  cluster_sync();
  {
    // CTA `rank` reduces rows [r0, r0 + rows) of the tile over the S partials.
    constexpr int kVec = BN / 4;  // float4 per row
    const int rows = (kProjBM + splits - 1) / splits;
    const int r0 = rank * rows;
    const int r1 = min(kProjBM, r0 + rows);
    for (int item = threadIdx.x; item < (r1 - r0) * kVec; item += kProjThreads) {
      const int row = r0 + item / kVec;
      const int c = (item % kVec) * 4;
      const float* src = part + row * S::kPartStride + c;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < splits; ++q) {
        const float4 w = ld_cluster_f4(map_to_rank(src, static_cast<uint32_t>(q)));
        v.x += w.x;
        v.y += w.y;
        v.z += w.z;
        v.w += w.w;
      }
      const int grow = m0 + row;
      const int n = n0 + c;
      if (grow < M && n < Nout) {
        if (bias != nullptr) {
          v.x += bias[n];
          v.y += bias[n + 1];
          v.z += bias[n + 2];
          v.w += bias[n + 3];
        }
        if constexpr (kOutBf16) {
          uint2* dst = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(grow) * Nout + n);
          *dst = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + static_cast<size_t>(grow) * Nout + n);
          if (accumulate) {
            const float4 old = *dst;
            v.x += old.x;
            v.y += old.y;
            v.z += old.z;
            v.w += old.w;
          }
          *dst = v;
        }
      }
    }
  }
  // No CTA leaves (and frees its shared memory) while another still reads it.
  cluster_sync();

  // ---- teardown: every MMA the issuer started has finished -----------------
  if (threadIdx.x == 32) mbar_drain(&mma_done, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sqa
