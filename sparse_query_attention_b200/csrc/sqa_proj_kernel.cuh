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
// Design: one CTA per 128 x BN output tile, four warps.
//   warp 0 / one lane : TMA producer, 64-wide K slices of A and B into a
//                       4-stage ring (128-byte swizzle).
//   warp 1            : issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//                       accumulator from warp-uniform code (lane 0 issues),
//                       commits each stage back to the producer.
//   all four warps    : epilogue, TMEM -> registers (+C, +bias) -> global.
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
template <int BN, bool kOutBf16, bool kAMN, bool kBMN>
__global__ void __launch_bounds__(128, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const float* __restrict__ bias, void* __restrict__ y, int M, int K, int Nout, int accumulate) {
  static_assert(!kBMN || BN % 64 == 0, "MN-contiguous B needs BN in 64, 128, 256");
  using S = ProjSmem<BN>;
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  constexpr uint32_t kMnChunk = 64 * 128;  // one 64 x 64 MN-contiguous box
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kProjStages];
  __shared__ __align__(8) uint64_t empty_bar[kProjStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + kProjStages * S::kABytes;

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kProjBM;
  const int n0 = blockIdx.y * BN;
  const int num_kb = (K + kProjBK - 1) / kProjBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kProjStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = tmem_base;

  if (warp == 0 && lane == 0) {
    // TMA producer
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % kProjStages;
      const uint32_t ph = (kb / kProjStages) & 1;
      if (kb >= kProjStages && !mbar_wait(&empty_bar[s], ph ^ 1, &abort_flag)) break;
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
      ++issued;
    }
    // No copy may still be landing in shared memory when the CTA exits.
    for (int kb = issued > kProjStages ? issued - kProjStages : 0; kb < issued; ++kb)
      mbar_drain(&full_bar[kb % kProjStages], (kb / kProjStages) & 1);
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
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % kProjStages;
      const uint32_t ph = (kb / kProjStages) & 1;
      if (!mbar_wait(&full_bar[s], ph, &abort_flag)) break;
      tc_fence_after();
      const uint64_t ad = desc_advance(a_desc0, s * S::kABytes);
      const uint64_t bd = desc_advance(b_desc0, s * S::kBBytes);
#pragma unroll
      for (int kk = 0; kk < kProjBK / 16; ++kk)
        mma_ss_w(tacc, desc_advance(ad, kk * kAStep), desc_advance(bd, kk * kBStep), idesc, (kb | kk) != 0);
      mma_commit_w(&empty_bar[s]);
    }
    mma_commit_w(&acc_bar);
  }
  __syncwarp();

  // Epilogue: warp w reads TMEM lanes [32w, 32w + 32) = output rows.
  const bool ok = mbar_wait(&acc_bar, 0, &abort_flag);
  tc_fence_after();
  if (ok) {
    const int row = m0 + warp * 32 + lane;
    const uint32_t lane_addr = tacc + (static_cast<uint32_t>(warp * 32) << 16);
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
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(row) * Nout + n);
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
  }
  // The MMA warp always commits acc_bar, so this returns once every MMA it
  // issued has finished, also after an abort.
  if (!ok && threadIdx.x == 0) mbar_drain(&acc_bar, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tacc, kTmemCols);
  }
}

}  // namespace sqa
