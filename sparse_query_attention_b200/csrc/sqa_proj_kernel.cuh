// sqa_proj_kernel.cuh - the reduced-width projection GEMM on the sm_100a
// tensor cores:  Y[M, Nout] = X[M, K] * W[Nout, K]^T (+ bias).
//
// In Sparse Query Attention the query projection produces only H_q * d_head
// columns and the output projection consumes only H_q * d_head ("ReactiveAI/
// xSMQAT-m" model card, note on model size); the key/value projections keep
// H_kv * d_head.  All four are this one contraction.
//
// Design: one CTA per 128 x BN output tile, four warps.
//   warp 0 / one lane : TMA producer, 64-wide K slices of X and W into a
//                       4-stage ring (128-byte swizzle, K-major).
//   warp 1 / one lane : issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//                       accumulator, commits each stage back to the producer.
//   all four warps    : epilogue, TMEM -> registers (+bias) -> global.
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

template <int BN, bool kOutBf16>
__global__ void __launch_bounds__(128, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const float* __restrict__ bias, void* __restrict__ y, int M, int K, int Nout) {
  using S = ProjSmem<BN>;
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
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
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
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
      tma_load_2d(&tm_x, &full_bar[s], a_tiles + s * S::kABytes, kb * kProjBK, m0);
      tma_load_2d(&tm_w, &full_bar[s], b_tiles + s * S::kBBytes, kb * kProjBK, n0);
      ++issued;
    }
    // No copy may still be landing in shared memory when the CTA exits.
    for (int kb = issued > kProjStages ? issued - kProjStages : 0; kb < issued; ++kb)
      mbar_drain(&full_bar[kb % kProjStages], (kb / kProjStages) & 1);
  } else if (warp == 1) {
    // MMA issuer: the whole warp runs the loop (operands stay warp-uniform),
    // lane 0 issues.  Descriptors are built once and advanced by offsets.
    constexpr uint32_t idesc = idesc_bf16_f32(kProjBM, BN, 0, 0);
    const uint64_t a_desc0 = smem_desc(smem_addr(a_tiles), 16, 1024, kSw128);
    const uint64_t b_desc0 = smem_desc(smem_addr(b_tiles), 16, 1024, kSw128);
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % kProjStages;
      const uint32_t ph = (kb / kProjStages) & 1;
      if (!mbar_wait(&full_bar[s], ph, &abort_flag)) break;
      tc_fence_after();
      const uint64_t ad = desc_advance(a_desc0, s * S::kABytes);
      const uint64_t bd = desc_advance(b_desc0, s * S::kBBytes);
#pragma unroll
      for (int kk = 0; kk < kProjBK / 16; ++kk)
        mma_ss_w(tacc, desc_advance(ad, kk * 32), desc_advance(bd, kk * 32), idesc, (kb | kk) != 0);
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
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    }
  }
  // The MMA thread always commits acc_bar, so this returns once every MMA
  // it issued has finished, also after an abort.
  if (!ok && threadIdx.x == 0) mbar_drain(&acc_bar, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tacc, kTmemCols);
  }
}

}  // namespace sqa
