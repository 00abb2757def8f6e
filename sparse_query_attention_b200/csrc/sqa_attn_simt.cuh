// sqa_attn_simt.cuh - straightforward CUDA-core kernels for the SQA attention
// core and its gradient: one thread per query row (forward, dQ) or per key
// row (dK/dV), fp32 arithmetic, key/value tiles staged in shared memory.
// They fix the layouts and the head grouping j = h / G that the tensor-core
// kernels must reproduce.
#pragma once

#include "sqa_ptx.cuh"

namespace sqa {

constexpr int kSimtRows = 64;  // query (or key) rows per block

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Forward: one thread per (b, t, h); online softmax over keys in tiles of 64.
template <int D>
__global__ void __launch_bounds__(kSimtRows)
    attn_fwd_simt_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                         const __nv_bfloat16* __restrict__ v, void* __restrict__ out, int out_bf16,
                         float* __restrict__ lse, int N, int H_q, int H_kv, int causal, float scale) {
  __shared__ __nv_bfloat16 ks[kSimtRows][D];
  __shared__ __nv_bfloat16 vs[kSimtRows][D];
  const int b = blockIdx.z, h = blockIdx.y;
  const int G = H_q / H_kv, j = h / G;
  const int t = blockIdx.x * kSimtRows + threadIdx.x;
  const bool valid = t < N;
  float qr[D], acc[D];
  const size_t qoff = ((static_cast<size_t>(b) * N + (valid ? t : 0)) * H_q + h) * D;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = bf2f(q[qoff + c]) * scale;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int t_last = min(N - 1, static_cast<int>(blockIdx.x * kSimtRows + kSimtRows - 1));
  const int key_end = causal ? t_last + 1 : N;
  for (int u0 = 0; u0 < key_end; u0 += kSimtRows) {
    __syncthreads();
    for (int i = threadIdx.x; i < kSimtRows * D; i += kSimtRows) {
      const int r = i / D, c = i % D, u = u0 + r;
      const size_t off = ((static_cast<size_t>(b) * N + u) * H_kv + j) * D + c;
      ks[r][c] = u < N ? k[off] : __float2bfloat16(0.f);
      vs[r][c] = u < N ? v[off] : __float2bfloat16(0.f);
    }
    __syncthreads();
    if (!valid) continue;
    for (int r = 0; r < kSimtRows; ++r) {
      const int u = u0 + r;
      if (u >= N || (causal && u > t)) break;
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) s = fmaf(qr[c], bf2f(ks[r][c]), s);
      const float m_new = fmaxf(m, s);
      const float corr = __expf(m - m_new);
      const float p = __expf(s - m_new);
      l = l * corr + p;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(acc[c], corr, p * bf2f(vs[r][c]));
      m = m_new;
    }
  }
  if (!valid) return;
  const float inv = 1.f / l;
  const size_t ooff = ((static_cast<size_t>(b) * N + t) * H_q + h) * D;
  if (out_bf16) {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
#pragma unroll
    for (int c = 0; c < D; ++c) o[ooff + c] = __float2bfloat16_rn(acc[c] * inv);
  } else {
    float* o = static_cast<float*>(out);
#pragma unroll
    for (int c = 0; c < D; ++c) o[ooff + c] = acc[c] * inv;
  }
  if (lse != nullptr) lse[(static_cast<size_t>(b) * H_q + h) * N + t] = m + logf(l);
}

// D_t = sum_c dO[t,c] * O[t,c], one warp per (b, t, h) row.
template <int D>
__global__ void attn_bwd_dot_kernel(const void* __restrict__ o, int o_bf16, const __nv_bfloat16* __restrict__ dout,
                                    float* __restrict__ dsum, int B, int N, int H_q) {
  const size_t row = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  const size_t rows = static_cast<size_t>(B) * N * H_q;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < D; c += 32) {
    const float ov = o_bf16 ? bf2f(static_cast<const __nv_bfloat16*>(o)[row * D + c])
                            : static_cast<const float*>(o)[row * D + c];
    acc = fmaf(ov, bf2f(dout[row * D + c]), acc);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    // row = (b * N + t) * H_q + h  ->  dsum[b, h, t]
    const int h = static_cast<int>(row % H_q);
    const size_t bt = row / H_q;
    const int t = static_cast<int>(bt % N);
    const int b = static_cast<int>(bt / N);
    dsum[(static_cast<size_t>(b) * H_q + h) * N + t] = acc;
  }
}

template <typename T>
__device__ __forceinline__ void store_val(T* p, float x);
template <>
__device__ __forceinline__ void store_val<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_val<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// dQ: one thread per (b, t, h); dq = scale * sum_u P (dP - D) k_u.
template <int D, typename GradT>
__global__ void __launch_bounds__(kSimtRows)
    attn_bwd_dq_simt_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                            const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                            const float* __restrict__ lse, const float* __restrict__ dsum, GradT* __restrict__ dq,
                            int N, int H_q, int H_kv, int causal, float scale) {
  __shared__ __nv_bfloat16 ks[kSimtRows][D];
  __shared__ __nv_bfloat16 vs[kSimtRows][D];
  const int b = blockIdx.z, h = blockIdx.y;
  const int G = H_q / H_kv, j = h / G;
  const int t = blockIdx.x * kSimtRows + threadIdx.x;
  const bool valid = t < N;
  float qr[D], gr[D], acc[D];
  const size_t off = ((static_cast<size_t>(b) * N + (valid ? t : 0)) * H_q + h) * D;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = bf2f(q[off + c]) * scale;
    gr[c] = bf2f(dout[off + c]);
    acc[c] = 0.f;
  }
  const size_t row_stat = (static_cast<size_t>(b) * H_q + h) * N + (valid ? t : 0);
  const float L = lse[row_stat], Dt = dsum[row_stat];
  const int t_last = min(N - 1, static_cast<int>(blockIdx.x * kSimtRows + kSimtRows - 1));
  const int key_end = causal ? t_last + 1 : N;
  for (int u0 = 0; u0 < key_end; u0 += kSimtRows) {
    __syncthreads();
    for (int i = threadIdx.x; i < kSimtRows * D; i += kSimtRows) {
      const int r = i / D, c = i % D, u = u0 + r;
      const size_t o2 = ((static_cast<size_t>(b) * N + u) * H_kv + j) * D + c;
      ks[r][c] = u < N ? k[o2] : __float2bfloat16(0.f);
      vs[r][c] = u < N ? v[o2] : __float2bfloat16(0.f);
    }
    __syncthreads();
    if (!valid) continue;
    for (int r = 0; r < kSimtRows; ++r) {
      const int u = u0 + r;
      if (u >= N || (causal && u > t)) break;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        s = fmaf(qr[c], bf2f(ks[r][c]), s);
        dp = fmaf(gr[c], bf2f(vs[r][c]), dp);
      }
      const float ds = __expf(s - L) * (dp - Dt);
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(ds, bf2f(ks[r][c]), acc[c]);
    }
  }
  if (!valid) return;
#pragma unroll
  for (int c = 0; c < D; ++c) store_val(dq + off + c, acc[c] * scale);
}

// dK, dV: one thread per (b, u, j); sums over the G query heads of group j
// and over the queries that see key u.
template <int D, typename GradT>
__global__ void __launch_bounds__(kSimtRows)
    attn_bwd_dkdv_simt_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                              const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                              const float* __restrict__ lse, const float* __restrict__ dsum,
                              GradT* __restrict__ dk, GradT* __restrict__ dv, int N, int H_q, int H_kv, int causal,
                              float scale) {
  __shared__ __nv_bfloat16 qs[kSimtRows][D];
  __shared__ __nv_bfloat16 gs[kSimtRows][D];
  __shared__ float ls[kSimtRows], ds_[kSimtRows];
  const int b = blockIdx.z, j = blockIdx.y;
  const int G = H_q / H_kv;
  const int u = blockIdx.x * kSimtRows + threadIdx.x;
  const bool valid = u < N;
  float kr[D], vr[D], ak[D], av[D];
  const size_t off = ((static_cast<size_t>(b) * N + (valid ? u : 0)) * H_kv + j) * D;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    kr[c] = bf2f(k[off + c]) * scale;
    vr[c] = bf2f(v[off + c]);
    ak[c] = 0.f;
    av[c] = 0.f;
  }
  const int t_begin = causal ? static_cast<int>(blockIdx.x * kSimtRows) : 0;
  for (int g = 0; g < G; ++g) {
    const int h = j * G + g;
    for (int t0 = t_begin; t0 < N; t0 += kSimtRows) {
      __syncthreads();
      for (int i = threadIdx.x; i < kSimtRows * D; i += kSimtRows) {
        const int r = i / D, c = i % D, t = t0 + r;
        const size_t o2 = ((static_cast<size_t>(b) * N + t) * H_q + h) * D + c;
        qs[r][c] = t < N ? q[o2] : __float2bfloat16(0.f);
        gs[r][c] = t < N ? dout[o2] : __float2bfloat16(0.f);
      }
      if (threadIdx.x < kSimtRows) {
        const int t = t0 + threadIdx.x;
        const size_t rs = (static_cast<size_t>(b) * H_q + h) * N + t;
        ls[threadIdx.x] = t < N ? lse[rs] : 0.f;
        ds_[threadIdx.x] = t < N ? dsum[rs] : 0.f;
      }
      __syncthreads();
      if (!valid) continue;
      for (int r = 0; r < kSimtRows; ++r) {
        const int t = t0 + r;
        if (t >= N) break;
        if (causal && t < u) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) {
          s = fmaf(bf2f(qs[r][c]), kr[c], s);
          dp = fmaf(bf2f(gs[r][c]), vr[c], dp);
        }
        const float p = __expf(s - ls[r]);
        const float ds = p * (dp - ds_[r]);
#pragma unroll
        for (int c = 0; c < D; ++c) {
          av[c] = fmaf(p, bf2f(gs[r][c]), av[c]);
          ak[c] = fmaf(ds, bf2f(qs[r][c]), ak[c]);
        }
      }
    }
  }
  if (!valid) return;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    store_val(dk + off + c, ak[c] * scale);
    store_val(dv + off + c, av[c]);
  }
}

}  // namespace sqa
