// sqa_api.cu - the C ABI declared in include/sqa.h: argument checks, TMA
// tensor-map encoding, kernel selection and launch.  One translation unit so
// the device status word and every kernel live in the same module.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "sqa.h"
#include "sqa_bwd_kernel.cuh"
#include "sqa_decode_kernel.cuh"
#include "sqa_fwd_kernel.cuh"
#include "sqa_fwd_quad_kernel.cuh"
#include "sqa_fwd_split_kernel.cuh"
#include "sqa_plan.h"
#include "sqa_proj_kernel.cuh"
#include "sqa_ptx.cuh"

namespace {

using sqa::kProjBM;
using sqa::plan::cluster_split;
using sqa::plan::decode_plan;
using sqa::plan::DecodePlan;
using sqa::plan::gemm_group_m;
using sqa::plan::head_pack;

// ---------------------------------------------------------------------------
// Driver entry point for cuTensorMapEncodeTiled, fetched once through the
// runtime (no link-time dependency on libcuda).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encode_fn_ready() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// A bf16 tensor map of rank `rank`; dims/strides innermost first, strides in
// bytes for dims 1.., box in elements, 128-byte swizzle unless given.
bool make_map_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box,
                   CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!encode_fn_ready()) return false;
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
                        reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides_bytes),
                        reinterpret_cast<const cuuint32_t*>(box), elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

sqa_status_t launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

// Every kernel of the library is launched with programmatic stream
// serialization: it may be scheduled while the previous kernel on the stream
// finishes, runs its set-up (barriers, TMEM allocation, descriptor
// prefetch) meanwhile, and waits in grid_dependency_wait for that kernel to
// complete before it touches global memory.  Stream order is kept for
// everything the kernels read and write.
template <typename... KArgs, typename... Args>
sqa_status_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

// launch_k for a grid of thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
sqa_status_t launch_k_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? SQA_OK : SQA_ERR_CUDA;
}

// How many clusters of `cluster` CTAs of `kern` (`threads` per CTA, `smem`
// bytes of dynamic shared memory, already allowed by cudaFuncSetAttribute)
// the current device runs at once.  Queried once per device, kernel and
// cluster size; 0 when the query fails.
int max_active_clusters(const void* kern, int cluster, int threads, int smem) {
  struct Entry {
    int dev;
    const void* kern;
    int cluster;
    int n;
  };
  static Entry cache[128];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].kern == kern && cache[i].cluster == cluster) return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(cluster * 64);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 0) n = 0;
  if (used < 128) cache[used++] = {dev, kern, cluster, n};
  return n;
}

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Streaming multiprocessors of the current device (looked up per call; the
// attribute query is cheap and the current device may change).
constexpr int kMaxDevices = 64;  // device ordinals with per-device host caches

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

sqa_status_t check_attn_args(const void* q, const void* k, const void* v, int B, int N, int H_q, int H_kv, int d,
                             float scale) {
  if (!q || !k || !v) return SQA_ERR_INVALID_ARG;
  if (B <= 0 || N <= 0 || H_q <= 0 || H_kv <= 0 || H_kv > H_q || H_q % H_kv != 0) return SQA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return SQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SQA_ERR_INVALID_ARG;
  if (d <= 0) return SQA_ERR_INVALID_ARG;
  if (!supported_d(d)) return SQA_ERR_UNSUPPORTED;
  // Row indices are formed in 32-bit arithmetic inside the kernels.
  if (static_cast<long long>(B) * N * H_q > (1ll << 31) - 1) return SQA_ERR_UNSUPPORTED;
  return SQA_OK;
}

// Key/value length: any positive length without a mask (cross / memory
// attention); a causal or windowed mask needs as many keys as queries.
sqa_status_t check_kv_length(int B, int N, int Nkv, int H_kv, int masked) {
  if (Nkv <= 0) return SQA_ERR_INVALID_ARG;
  if (masked && Nkv != N) return SQA_ERR_INVALID_ARG;
  // Band arithmetic (t + win_r + 1 with win_r <= N) stays in 32 bits.
  if (masked && N > (1 << 30)) return SQA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Nkv * H_kv > (1ll << 31) - 1) return SQA_ERR_UNSUPPORTED;
  return SQA_OK;
}

// Shape, mask and token strides of one attention call.  A token stride is
// the number of elements from one token's row of heads to the next: H * d for
// the dense layouts, (H_q + 2 H_kv) * d inside a packed QKV buffer.
struct AttnDesc {
  int B, N, Nkv, H_q, H_kv, d;
  int masked;         // band mask: t - win_l <= u <= t + win_r
  int win_l, win_r;   // clamped to N; causal is (N, 0)
  int longest_first;  // masked problems: schedule the last token blocks first
  float scale;
  long long ld_q, ld_kv;    // Q; K and V
  long long ld_dq, ld_dkv;  // dQ; dK and dV (backward only)
};

AttnDesc dense_desc(int B, int N, int Nkv, int H_q, int H_kv, int d, int causal, float scale) {
  AttnDesc a;
  a.B = B;
  a.N = N;
  a.Nkv = Nkv;
  a.H_q = H_q;
  a.H_kv = H_kv;
  a.d = d;
  a.masked = causal ? 1 : 0;
  a.win_l = N;
  a.win_r = 0;
  a.longest_first = a.masked;
  a.scale = scale;
  a.ld_q = a.ld_dq = static_cast<long long>(H_q) * d;
  a.ld_kv = a.ld_dkv = static_cast<long long>(H_kv) * d;
  return a;
}

// The packed layout [B, N, H_q + 2 H_kv, d]: Q heads, then K, then V.
AttnDesc packed_desc(int B, int N, int H_q, int H_kv, int d, int causal, float scale) {
  AttnDesc a = dense_desc(B, N, N, H_q, H_kv, d, causal, scale);
  a.ld_q = a.ld_kv = a.ld_dq = a.ld_dkv = static_cast<long long>(H_q + 2 * H_kv) * d;
  return a;
}

// Sliding window: query t sees keys t - left <= u <= t + right.  Sides of
// N or more are unbounded, so (>= N, 0) is the causal mask.
AttnDesc window_desc(int B, int N, int H_q, int H_kv, int d, int left, int right, float scale) {
  AttnDesc a = dense_desc(B, N, N, H_q, H_kv, d, 1, scale);
  a.win_l = left < N ? left : N;
  a.win_r = right < N ? right : N;
  a.longest_first = a.win_r == 0 && a.win_l == N;
  return a;
}

sqa_status_t check_desc(const void* q, const void* k, const void* v, const AttnDesc& a) {
  sqa_status_t s = check_attn_args(q, k, v, a.B, a.N, a.H_q, a.H_kv, a.d, a.scale);
  if (s != SQA_OK) return s;
  s = check_kv_length(a.B, a.N, a.Nkv, a.H_kv, a.masked);
  if (s != SQA_OK) return s;
  if (a.win_l < 0 || a.win_r < 0) return SQA_ERR_INVALID_ARG;
  // Token rows are whole 16-byte units (a TMA stride rule) and the element
  // offsets of the last token of the last batch fit in 32-bit row arithmetic.
  const long long lds[4] = {a.ld_q, a.ld_kv, a.ld_dq, a.ld_dkv};
  for (long long ld : lds)
    if (ld % 8 != 0) return SQA_ERR_INVALID_ARG;
  if (a.ld_q < static_cast<long long>(a.H_q) * a.d || a.ld_dq < static_cast<long long>(a.H_q) * a.d ||
      a.ld_kv < static_cast<long long>(a.H_kv) * a.d || a.ld_dkv < static_cast<long long>(a.H_kv) * a.d)
    return SQA_ERR_INVALID_ARG;
  return SQA_OK;
}

// ---------------------------------------------------------------------------
// Attention forward
// ---------------------------------------------------------------------------
CUtensorMapSwizzle tma_swizzle_for_row_bytes(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}


template <int D>
sqa_status_t launch_fwd_tc(const void* q, const void* k, const void* v, void* out, int out_bf16, float* lse,
                           const AttnDesc& a, cudaStream_t st) {
  using C = sqa::FwdCfg<D>;
  const int B = a.B, N = a.N, Nkv = a.Nkv, H_q = a.H_q, H_kv = a.H_kv;
  const int G = H_q / H_kv;
  const int g = head_pack(G);
  int log2g = 0;
  while ((1 << log2g) < g) ++log2g;
  const int T = 128 / g;
  const CUtensorMapSwizzle swz = tma_swizzle_for_row_bytes(C::kRowBytes);
  CUtensorMap mq, mk, mv;
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(H_q), uint64_t(N), uint64_t(B)};
    const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(a.ld_q) * 2, uint64_t(N) * a.ld_q * 2};
    const uint32_t box[4] = {uint32_t(C::kRowElems), uint32_t(g), uint32_t(T), 1};
    if (!make_map_bf16(&mq, q, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(H_kv), uint64_t(Nkv), uint64_t(B)};
    const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(a.ld_kv) * 2, uint64_t(Nkv) * a.ld_kv * 2};
    const uint32_t box[4] = {uint32_t(C::kRowElems), 1, 128, 1};
    if (!make_map_bf16(&mk, k, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
    if (!make_map_bf16(&mv, v, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
  }
  sqa::FwdParams p;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.N = N;
  p.Nkv = Nkv;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.G = G;
  p.g = g;
  p.log2g = log2g;
  p.n_sub = G / g;
  p.n_tblk = (N + 2 * T - 1) / (2 * T);
  p.masked = a.masked;
  p.win_l = a.win_l;
  p.win_r = a.win_r;
  p.longest_first = a.longest_first;
  p.tblk0 = 0;
  p.wait_at_exit = 0;
  p.kv_splits = 1;
  p.out_bf16 = out_bf16;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const long long gy = static_cast<long long>(H_kv) * p.n_sub;
  if (gy > 65535 || B > 65535) return SQA_ERR_UNSUPPORTED;
  dim3 grid(p.n_tblk, static_cast<unsigned>(gy), B);
  if constexpr (D <= 64) {
    // Four virtual tiles (two key halves per query tile): see sqa_fwd_quad_kernel.cuh.
    auto kern = sqa::sqa_fwd_quad_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sqa::QuadCfg<D>::kSmemBytes) !=
        cudaSuccess)
      return SQA_ERR_CUDA;
    return launch_k(kern, grid, dim3(sqa::kQuadThreads), sqa::QuadCfg<D>::kSmemBytes, st, mq, mk, mv, p);
  } else {
    // The cover of the query tiles (two-tile grid, split grid, or both) is
    // sqa::plan::fwd_wave_plan (sqa_plan.h), after the key-range split below.
    const int sms = num_sms();
    if (sms <= 0) return SQA_ERR_CUDA;
    // Few query tiles against many keys (unmasked: cross attention from a
    // short query sequence, or small batches): split every token block's key
    // range over a cluster of 2, 4 or 8 two-tile CTAs, the largest for which
    // all clusters run at once and each CTA keeps at least four key blocks;
    // the CTAs merge their rows' partial results in distributed shared memory.
    // (A cluster's CTAs are consecutive along x, so the grid keeps its plain
    // order: unmasked problems never take the longest-first order.)
    if (!a.masked && !a.longest_first) {
      auto kern = sqa::sqa_fwd_kernel<D, true>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return SQA_ERR_CUDA;
      const long long units = static_cast<long long>(p.n_tblk) * gy * B;
      const int splits = cluster_split(units, (Nkv + 127) / 128, 4, 8, [&](int c) {
        return max_active_clusters(reinterpret_cast<const void*>(kern), c, sqa::kFwdThreads, C::kSmemBytes);
      });
      if (splits > 1) {
        p.kv_splits = splits;
        const dim3 grid_c(static_cast<unsigned>(p.n_tblk * splits), static_cast<unsigned>(gy), B);
        return launch_k_cluster(kern, grid_c, dim3(sqa::kFwdThreads), C::kSmemBytes, st, splits, mq, mk, mv, p);
      }
    }
    const int n_tiles = (N + T - 1) / T;
    const sqa::plan::FwdWavePlan cover = sqa::plan::fwd_wave_plan(p.n_tblk, gy * B, n_tiles, sms, a.masked);
    auto launch_split = [&](int tile0, int tiles) -> sqa_status_t {
      sqa::FwdParams ps = p;
      ps.n_tblk = n_tiles;
      ps.tblk0 = tile0;
      ps.wait_at_exit = tile0 > 0;  // after the two-tile launch of the same problem
      dim3 grid1(tiles, static_cast<unsigned>(gy), B);
      auto kern = sqa::sqa_fwd_split_kernel<D>;
      constexpr int smem = sqa::SplitCfg<D>::kSmemBytes;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SQA_ERR_CUDA;
      return launch_k(kern, grid1, dim3(sqa::kFwdThreads), smem, st, mq, mk, mv, ps);
    };
    if (cover.cover == sqa::plan::FwdCover::kSplit) return launch_split(0, n_tiles);
    if (cover.cover == sqa::plan::FwdCover::kMixed) {
      auto kern = sqa::sqa_fwd_kernel<D>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return SQA_ERR_CUDA;
      dim3 grid_a(cover.n_a, static_cast<unsigned>(gy), B);
      const sqa_status_t s2 = launch_k(kern, grid_a, dim3(sqa::kFwdThreads), C::kSmemBytes, st, mq, mk, mv, p);
      if (s2 != SQA_OK) return s2;
      return launch_split(2 * cover.n_a, n_tiles - 2 * cover.n_a);
    }
    auto kern = sqa::sqa_fwd_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return SQA_ERR_CUDA;
    return launch_k(kern, grid, dim3(sqa::kFwdThreads), C::kSmemBytes, st, mq, mk, mv, p);
  }
}

sqa_status_t attn_fwd_impl(const void* q, const void* k, const void* v, void* out, sqa_dtype_t out_dtype, float* lse,
                           const AttnDesc& a, void* stream) {
  sqa_status_t s = check_desc(q, k, v, a);
  if (s != SQA_OK) return s;
  if (!out || !aligned16(out) || (lse && !aligned16(lse))) return SQA_ERR_INVALID_ARG;
  if (out_dtype != SQA_DT_F32 && out_dtype != SQA_DT_BF16) return SQA_ERR_INVALID_ARG;
  const int ob = out_dtype == SQA_DT_BF16;
  cudaStream_t st = as_stream(stream);
  switch (a.d) {
    case 16: return launch_fwd_tc<16>(q, k, v, out, ob, lse, a, st);
    case 32: return launch_fwd_tc<32>(q, k, v, out, ob, lse, a, st);
    case 64: return launch_fwd_tc<64>(q, k, v, out, ob, lse, a, st);
    default: return launch_fwd_tc<128>(q, k, v, out, ob, lse, a, st);
  }
}

// ---------------------------------------------------------------------------
// Attention backward
// ---------------------------------------------------------------------------
// Workspace: D and LSE*log2(e), each [B, H_q, n_pad] fp32, n_pad = N rounded
// up to 128 so every tile the kernels touch is in bounds.
int bwd_n_pad(int N) { return (N + 127) / 128 * 128; }

size_t bwd_half_bytes(int B, int N, int H_q) {
  const size_t rows = static_cast<size_t>(B) * H_q * bwd_n_pad(N);
  return ((rows * sizeof(float)) + 255) & ~size_t(255);
}

size_t bwd_workspace_bytes(int B, int N, int H_q) { return 2 * bwd_half_bytes(B, N, H_q); }

bool make_map_f32_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner) {
  if (!encode_fn_ready()) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {box_inner, 1};
  const cuuint32_t es[2] = {1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [B, N, H, D] viewed as the 4-D map {D, H, N, B}, box {row, heads, tokens, 1}.
// ld: elements from one token to the next (H * D when dense).
template <int D>
bool make_map_bnhd(CUtensorMap* map, const void* base, int B, int N, int H, long long ld, uint32_t box_heads,
                   uint32_t box_tokens) {
  constexpr int kRowElems = D < 64 ? D : 64;
  const uint64_t dims[4] = {uint64_t(D), uint64_t(H), uint64_t(N), uint64_t(B)};
  const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(ld) * 2, uint64_t(N) * ld * 2};
  const uint32_t box[4] = {uint32_t(kRowElems), box_heads, box_tokens, 1};
  return make_map_bf16(map, base, 4, dims, strides, box, tma_swizzle_for_row_bytes(kRowElems * 2));
}

template <int D, typename GradT>
sqa_status_t launch_bwd_tc(const void* q, const void* k, const void* v, const void* o, int o_bf16, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, const AttnDesc& a, void* workspace,
                           cudaStream_t st) {
  const int B = a.B, N = a.N, Nkv = a.Nkv, H_q = a.H_q, H_kv = a.H_kv;
  const int n_pad = bwd_n_pad(N);
  float* dsum = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + bwd_half_bytes(B, N, H_q));
  const int G = H_q / H_kv;
  const int g = head_pack(G);
  int log2g = 0;
  while ((1 << log2g) < g) ++log2g;
  const int T = 128 / g;

  sqa::BwdParams p;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dsum = dsum;
  p.lse2 = lse2;
  p.B = B;
  p.N = N;
  p.Nkv = Nkv;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.G = G;
  p.n_pad = n_pad;
  p.g = g;
  p.log2g = log2g;
  p.n_sub = G / g;
  p.n_tblk = (N + T - 1) / T;
  p.masked = a.masked;
  p.win_l = a.win_l;
  p.win_r = a.win_r;
  p.longest_first = a.longest_first;
  p.kv_splits = 1;
  p.wait_at_exit = 0;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ld_dq = static_cast<int>(a.ld_dq);
  p.ld_dkv = static_cast<int>(a.ld_dkv);
  const long long gy = static_cast<long long>(H_kv) * p.n_sub;
  if (gy > 65535 || B > 65535) return SQA_ERR_UNSUPPORTED;

  CUtensorMap m_k128, m_v128, m_q64, m_do64, m_l2, m_ds, m_qp, m_dop, m_k64, m_v64;
  const long long ld_do = static_cast<long long>(H_q) * D;  // dO is always dense
  if (!make_map_bnhd<D>(&m_k128, k, B, Nkv, H_kv, a.ld_kv, 1, 128) ||
      !make_map_bnhd<D>(&m_v128, v, B, Nkv, H_kv, a.ld_kv, 1, 128) ||
      !make_map_bnhd<D>(&m_q64, q, B, N, H_q, a.ld_q, 1, 64) ||
      !make_map_bnhd<D>(&m_do64, dout, B, N, H_q, ld_do, 1, 64) ||
      !make_map_bnhd<D>(&m_qp, q, B, N, H_q, a.ld_q, g, T) || !make_map_bnhd<D>(&m_dop, dout, B, N, H_q, ld_do, g, T) ||
      !make_map_bnhd<D>(&m_k64, k, B, Nkv, H_kv, a.ld_kv, 1, 64) ||
      !make_map_bnhd<D>(&m_v64, v, B, Nkv, H_kv, a.ld_kv, 1, 64) ||
      !make_map_f32_2d(&m_l2, lse2, n_pad, uint64_t(B) * H_q, 64) ||
      !make_map_f32_2d(&m_ds, dsum, n_pad, uint64_t(B) * H_q, 64))
    return SQA_ERR_CUDA;

  // 1. D and LSE in log2 units.
  const size_t prep_rows = static_cast<size_t>(B) * H_q * n_pad;
  sqa_status_t s = launch_k(sqa::bwd_prep_kernel<D>, dim3(static_cast<unsigned>((prep_rows * (D / 8) + 255) / 256)),
                            dim3(256), 0, st, o, o_bf16, static_cast<const __nv_bfloat16*>(dout), lse, dsum, lse2, B,
                            N, H_q, n_pad);
  if (s != SQA_OK) return s;

  // 2. dK, dV (KV-outer).  The statistics ride in the score MMAs unless
  // 1 / (scale log2 e) is out of range (a zero or near-zero scale).
  {
    const bool fold = std::fabs(p.scale_log2) >= 1e-30f;
    auto kern = fold ? sqa::bwd_dkdv_kernel<D, GradT, true> : sqa::bwd_dkdv_kernel<D, GradT, false>;
    constexpr int smem = sqa::DkdvCfg<D>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return SQA_ERR_CUDA;
    // Unmasked problems whose key tiles leave SMs idle (cross / memory
    // attention over a short key sequence) split each tile's steps over a
    // cluster of 2, 4 or 8 CTAs: the largest split for which every cluster
    // runs at once and each CTA keeps at least 8 of the tile's steps.  A grid
    // that already fills the SMs is left whole (more, shorter CTAs in several
    // waves measured no faster).  The split is an instantiation of its own
    // (with the statistics folded), so the unsplit kernel keeps its code.
    const long long units = static_cast<long long>((Nkv + 127) / 128) * H_kv * B;
    const long long n_all = static_cast<long long>(G) * ((N + 63) / 64);
    int splits = 1;
    if (fold && !a.masked && !a.longest_first) {
      auto kern_s = sqa::bwd_dkdv_kernel<D, GradT, true, true>;
      if (cudaFuncSetAttribute(kern_s, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SQA_ERR_CUDA;
      splits = cluster_split(units, n_all, 8, 8, [&](int c) {
        return max_active_clusters(reinterpret_cast<const void*>(kern_s), c, sqa::kBwdThreads, smem);
      });
    }
    p.kv_splits = splits;
    dim3 grid(static_cast<unsigned>(((Nkv + 127) / 128) * splits), H_kv, B);
    s = splits > 1 ? launch_k_cluster(sqa::bwd_dkdv_kernel<D, GradT, true, true>, grid, dim3(sqa::kBwdThreads), smem,
                                      st, splits, m_k128, m_v128, m_q64, m_do64, m_l2, m_ds, p)
                   : launch_k(kern, grid, dim3(sqa::kBwdThreads), smem, st, m_k128, m_v128, m_q64, m_do64, m_l2,
                              m_ds, p);
    if (s != SQA_OK) return s;
    p.kv_splits = 1;
  }
  // 3. dQ (Q-outer).  Unmasked problems whose query tiles leave SMs idle
  // (few queries against many keys) split each tile's key sub-tiles over a
  // cluster of 2, 4 or 8 CTAs, as dK/dV does its steps.
  {
    auto kern = sqa::bwd_dq_kernel<D, GradT>;
    constexpr int smem = sqa::DqCfg<D>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return SQA_ERR_CUDA;
    int splits = 1;
    if (!a.masked && !a.longest_first) {
      auto kern_s = sqa::bwd_dq_kernel<D, GradT, true>;
      if (cudaFuncSetAttribute(kern_s, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SQA_ERR_CUDA;
      const long long units = static_cast<long long>(p.n_tblk) * gy * B;
      const long long n_all = (Nkv + 63) / 64;
      splits = cluster_split(units, n_all, 8, 8, [&](int c) {
        return max_active_clusters(reinterpret_cast<const void*>(kern_s), c, sqa::kBwdThreads, smem);
      });
    }
    p.kv_splits = splits;
    p.wait_at_exit = 1;  // follows dK/dV on the stream and reads nothing it writes
    dim3 grid(static_cast<unsigned>(p.n_tblk * splits), static_cast<unsigned>(gy), B);
    if (splits > 1)
      return launch_k_cluster(sqa::bwd_dq_kernel<D, GradT, true>, grid, dim3(sqa::kBwdThreads), smem, st, splits,
                              m_qp, m_dop, m_k64, m_v64, p);
    return launch_k(kern, grid, dim3(sqa::kBwdThreads), smem, st, m_qp, m_dop, m_k64, m_v64, p);
  }
}

template <int D>
sqa_status_t launch_bwd_d(bool grad_bf16, const void* q, const void* k, const void* v, const void* o, int o_bf16,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, const AttnDesc& a,
                          void* ws, cudaStream_t st) {
  if (grad_bf16)
    return launch_bwd_tc<D, __nv_bfloat16>(q, k, v, o, o_bf16, dout, lse, dq, dk, dv, a, ws, st);
  return launch_bwd_tc<D, float>(q, k, v, o, o_bf16, dout, lse, dq, dk, dv, a, ws, st);
}

sqa_status_t attn_bwd_impl(const void* q, const void* k, const void* v, const void* out, sqa_dtype_t o_dtype,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                           const AttnDesc& a, void* workspace, size_t workspace_bytes, void* stream) {
  sqa_status_t s = check_desc(q, k, v, a);
  if (s != SQA_OK) return s;
  if (!out || !dout || !lse || !dq || !dk || !dv || !workspace) return SQA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(lse) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(workspace))
    return SQA_ERR_INVALID_ARG;
  if ((o_dtype != SQA_DT_F32 && o_dtype != SQA_DT_BF16) || (grad_dtype != SQA_DT_F32 && grad_dtype != SQA_DT_BF16))
    return SQA_ERR_INVALID_ARG;
  if (workspace_bytes < bwd_workspace_bytes(a.B, a.N, a.H_q)) return SQA_ERR_INVALID_ARG;
  const bool gb = grad_dtype == SQA_DT_BF16;
  const int ob = o_dtype == SQA_DT_BF16;
  cudaStream_t st = as_stream(stream);
  switch (a.d) {
    case 16: return launch_bwd_d<16>(gb, q, k, v, out, ob, dout, lse, dq, dk, dv, a, workspace, st);
    case 32: return launch_bwd_d<32>(gb, q, k, v, out, ob, dout, lse, dq, dk, dv, a, workspace, st);
    case 64: return launch_bwd_d<64>(gb, q, k, v, out, ob, dout, lse, dq, dk, dv, a, workspace, st);
    default: return launch_bwd_d<128>(gb, q, k, v, out, ob, dout, lse, dq, dk, dv, a, workspace, st);
  }
}

// ---------------------------------------------------------------------------
// Projection GEMM
// ---------------------------------------------------------------------------

template <int BN, bool kBf16, bool kAMN, bool kBMN>
sqa_status_t launch_gemm_bn(const CUtensorMap& ma, const CUtensorMap& mb, const float* bias, void* c, int M, int N,
                            int K, int accumulate, cudaStream_t st) {
  auto kern = sqa::proj_gemm_kernel<BN, kBf16, kAMN, kBMN>;
  constexpr int smem = sqa::ProjSmem<BN>::kDynamicBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SQA_ERR_CUDA;
  // Persistent: one CTA per SM (or per tile when there are fewer tiles).
  const long long tiles = static_cast<long long>((M + kProjBM - 1) / kProjBM) * ((N + BN - 1) / BN);
  const int sms = num_sms();
  if (sms <= 0) return SQA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  return launch_k(kern, dim3(grid), dim3(sqa::kProjThreads), smem, st, ma, mb, bias, c, M, K, N, accumulate,
                  gemm_group_m(M, N, K, kProjBM));
}

// CTA-pair GEMM (K-contiguous A and B): clusters of two, persistent over the
// 256 x 256 output tiles, as many pairs as can be resident at once.
template <bool kBf16>
sqa_status_t launch_gemm_pair(const CUtensorMap& ma, const CUtensorMap& mb, const float* bias, void* c, int M, int N,
                              int K, int accumulate, cudaStream_t st) {
  auto kern = sqa::proj_gemm_pair_kernel<kBf16>;
  constexpr int smem = sqa::kPairDynamicBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SQA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(sqa::kProjThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_pairs = 0;
  cfg.gridDim = dim3(2 * 64);
  if (cudaOccupancyMaxActiveClusters(&max_pairs, kern, &cfg) != cudaSuccess || max_pairs <= 0) return SQA_ERR_CUDA;
  const long long tiles = static_cast<long long>((M + 2 * kProjBM - 1) / (2 * kProjBM)) *
                          ((N + sqa::kPairBN - 1) / sqa::kPairBN);
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  const int group_m = gemm_group_m(M, N, K, 2 * kProjBM);
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, bias, c, M, K, N, accumulate, group_m) == cudaSuccess
             ? SQA_OK
             : SQA_ERR_CUDA;
}

// Split K over clusters (proj_gemm_splitk_kernel): for products with few
// output tiles and a long K.  Clusters of 16 (a non-portable size, allowed
// where the device runs it), 8, 4 or 2 CTAs: the largest for which one
// cluster per output tile fits on the device at once and each CTA keeps at
// least four K blocks; 0 when none does.
template <int BN, bool kBf16, bool kAMN, bool kBMN>
int gemm_split_count(long long tiles, int num_kb) {
  auto kern = sqa::proj_gemm_splitk_kernel<BN, kBf16, kAMN, kBMN>;
  constexpr int smem = sqa::SplitSmem<BN>::kDynamicBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
  const bool wide = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  const int splits = cluster_split(tiles, num_kb, 4, wide ? 16 : 8, [&](int c) {
    return max_active_clusters(reinterpret_cast<const void*>(kern), c, sqa::kProjThreads, smem);
  });
  return splits > 1 ? splits : 0;
}

template <int BN, bool kBf16, bool kAMN, bool kBMN>
sqa_status_t launch_gemm_splitk(const CUtensorMap& ma, const CUtensorMap& mb, const float* bias, void* c, int M,
                                int N, int K, int accumulate, int splits, cudaStream_t st) {
  auto kern = sqa::proj_gemm_splitk_kernel<BN, kBf16, kAMN, kBMN>;
  constexpr int smem = sqa::SplitSmem<BN>::kDynamicBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SQA_ERR_CUDA;
  const long long tiles = static_cast<long long>((M + kProjBM - 1) / kProjBM) * ((N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * splits));
  cfg.blockDim = dim3(sqa::kProjThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, bias, c, M, K, N, accumulate) == cudaSuccess ? SQA_OK
                                                                                              : SQA_ERR_CUDA;
}

// Split-K dispatch for one layout pair: BN = 64, or 32 for a K-contiguous B
// of at most 32 columns.  Sets *taken when it launched (or failed to).
template <bool kAMN, bool kBMN>
sqa_status_t gemm_splitk_layout(const void* a, const void* b, const uint64_t* a_dims, const uint64_t* a_strides,
                                const uint32_t* a_box, const uint64_t* b_dims, const uint64_t* b_strides,
                                const float* bias, void* c, bool bf, int M, int N, int K, int accumulate,
                                cudaStream_t st, bool* taken) {
  *taken = false;
  const int bn = (!kBMN && N <= 32) ? 32 : 64;
  const long long tiles = static_cast<long long>((M + kProjBM - 1) / kProjBM) * ((N + bn - 1) / bn);
  const int num_kb = (K + sqa::kProjBK - 1) / sqa::kProjBK;
  int splits = 0;
  if (bn == 32) {
    if constexpr (!kBMN)
      splits = bf ? gemm_split_count<32, true, kAMN, kBMN>(tiles, num_kb)
                  : gemm_split_count<32, false, kAMN, kBMN>(tiles, num_kb);
  } else {
    splits = bf ? gemm_split_count<64, true, kAMN, kBMN>(tiles, num_kb)
                : gemm_split_count<64, false, kAMN, kBMN>(tiles, num_kb);
  }
  if (splits < 2) return SQA_OK;
  *taken = true;
  CUtensorMap ma, mb;
  const uint32_t b_box[2] = {64, kBMN ? 64u : uint32_t(bn)};
  if (!make_map_bf16(&ma, a, 2, a_dims, a_strides, a_box) || !make_map_bf16(&mb, b, 2, b_dims, b_strides, b_box))
    return SQA_ERR_CUDA;
  if (bn == 32) {
    if constexpr (!kBMN)
      return bf ? launch_gemm_splitk<32, true, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, splits, st)
                : launch_gemm_splitk<32, false, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, splits, st);
    return SQA_ERR_UNSUPPORTED;
  }
  return bf ? launch_gemm_splitk<64, true, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, splits, st)
            : launch_gemm_splitk<64, false, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, splits, st);
}

template <bool kBf16, bool kAMN, bool kBMN>
sqa_status_t launch_gemm_layouts(const CUtensorMap& ma, const CUtensorMap& mb, int bn, const float* bias, void* c,
                                 int M, int N, int K, int accumulate, cudaStream_t st) {
  switch (bn) {
    case 16:
      if constexpr (!kBMN) return launch_gemm_bn<16, kBf16, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, st);
      break;
    case 32:
      if constexpr (!kBMN) return launch_gemm_bn<32, kBf16, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, st);
      break;
    case 64: return launch_gemm_bn<64, kBf16, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, st);
    case 128: return launch_gemm_bn<128, kBf16, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, st);
    default: return launch_gemm_bn<256, kBf16, kAMN, kBMN>(ma, mb, bias, c, M, N, K, accumulate, st);
  }
  return SQA_ERR_UNSUPPORTED;
}

// C[M, N] (+)= sum_k A(m, k) B(n, k) (+ bias) with A, B K- or MN-contiguous.
sqa_status_t gemm_impl(const void* a, bool a_mn, const void* b, bool b_mn, const float* bias, void* c,
                       sqa_dtype_t c_dtype, int accumulate, int M, int N, int K, void* stream) {
  if (!a || !b || !c) return SQA_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return SQA_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c) || (bias && !aligned16(bias))) return SQA_ERR_INVALID_ARG;
  if (c_dtype != SQA_DT_F32 && c_dtype != SQA_DT_BF16) return SQA_ERR_INVALID_ARG;
  if (accumulate && c_dtype != SQA_DT_F32) return SQA_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 16 != 0 || (a_mn && M % 16 != 0)) return SQA_ERR_UNSUPPORTED;
  // BN: the narrowest tile covering N, at most 256 (at least 64 when B is
  // MN-contiguous: its tiles are loaded as 64-column boxes).
  int bn = b_mn ? 64 : 16;
  while (bn < N && bn < 256) bn *= 2;
  CUtensorMap ma, mb;
  const uint64_t a_dims[2] = {uint64_t(a_mn ? M : K), uint64_t(a_mn ? K : M)};
  const uint64_t a_strides[1] = {uint64_t(a_mn ? M : K) * 2};
  const uint32_t a_box[2] = {64, a_mn ? 64u : uint32_t(kProjBM)};
  const uint64_t b_dims[2] = {uint64_t(b_mn ? N : K), uint64_t(b_mn ? K : N)};
  const uint64_t b_strides[1] = {uint64_t(b_mn ? N : K) * 2};
  const uint32_t b_box[2] = {64, b_mn ? 64u : uint32_t(bn)};
  cudaStream_t st = as_stream(stream);
  const bool bf = c_dtype == SQA_DT_BF16;
  const int sms = num_sms();
  // Few output tiles and a long K (a layer's weight gradients, K = tokens):
  // split K over clusters instead of leaving most SMs idle.
  const long long tiles = static_cast<long long>((M + kProjBM - 1) / kProjBM) * ((N + bn - 1) / bn);
  if (sms > 0 && tiles * 4 <= sms && (K + sqa::kProjBK - 1) / sqa::kProjBK >= 8) {
    bool taken = false;
    sqa_status_t r = SQA_OK;
    if (!a_mn && !b_mn)
      r = gemm_splitk_layout<false, false>(a, b, a_dims, a_strides, a_box, b_dims, b_strides, bias, c, bf, M, N, K,
                                           accumulate, st, &taken);
    else if (!a_mn && b_mn)
      r = gemm_splitk_layout<false, true>(a, b, a_dims, a_strides, a_box, b_dims, b_strides, bias, c, bf, M, N, K,
                                          accumulate, st, &taken);
    else if (a_mn && b_mn)
      r = gemm_splitk_layout<true, true>(a, b, a_dims, a_strides, a_box, b_dims, b_strides, bias, c, bf, M, N, K,
                                         accumulate, st, &taken);
    else
      r = gemm_splitk_layout<true, false>(a, b, a_dims, a_strides, a_box, b_dims, b_strides, bias, c, bf, M, N, K,
                                          accumulate, st, &taken);
    if (taken) return r;
  }
  if (!make_map_bf16(&ma, a, 2, a_dims, a_strides, a_box) || !make_map_bf16(&mb, b, 2, b_dims, b_strides, b_box))
    return SQA_ERR_CUDA;
  // Large K-contiguous products (the layer's forward projections, nn.Linear
  // layout) run on CTA pairs with 256 x 256 tiles when there are enough tiles
  // to occupy every pair of SMs.
  const long long pair_tiles = static_cast<long long>((M + 2 * kProjBM - 1) / (2 * kProjBM)) *
                               ((N + sqa::kPairBN - 1) / sqa::kPairBN);
  if (!a_mn && !b_mn && N >= sqa::kPairBN && sms > 0 && pair_tiles >= sms / 2) {
    CUtensorMap mb2;
    const uint32_t b2_box[2] = {64, uint32_t(kProjBM)};  // each CTA loads 128 of the tile's 256 B rows
    if (!make_map_bf16(&mb2, b, 2, b_dims, b_strides, b2_box)) return SQA_ERR_CUDA;
    return bf ? launch_gemm_pair<true>(ma, mb2, bias, c, M, N, K, accumulate, st)
              : launch_gemm_pair<false>(ma, mb2, bias, c, M, N, K, accumulate, st);
  }
  if (!a_mn && !b_mn)
    return bf ? launch_gemm_layouts<true, false, false>(ma, mb, bn, bias, c, M, N, K, accumulate, st)
              : launch_gemm_layouts<false, false, false>(ma, mb, bn, bias, c, M, N, K, accumulate, st);
  if (!a_mn && b_mn)
    return bf ? launch_gemm_layouts<true, false, true>(ma, mb, bn, bias, c, M, N, K, accumulate, st)
              : launch_gemm_layouts<false, false, true>(ma, mb, bn, bias, c, M, N, K, accumulate, st);
  if (a_mn && b_mn)
    return bf ? launch_gemm_layouts<true, true, true>(ma, mb, bn, bias, c, M, N, K, accumulate, st)
              : launch_gemm_layouts<false, true, true>(ma, mb, bn, bias, c, M, N, K, accumulate, st);
  return bf ? launch_gemm_layouts<true, true, false>(ma, mb, bn, bias, c, M, N, K, accumulate, st)
            : launch_gemm_layouts<false, true, false>(ma, mb, bn, bias, c, M, N, K, accumulate, st);
}

// ---------------------------------------------------------------------------
// KV-cache decode
// ---------------------------------------------------------------------------
// Chunking of the cache: sqa::plan::decode_plan (sqa_plan.h).

size_t decode_part_l_bytes(int n_split, int B, int n_new, int H_q) {
  const size_t n = static_cast<size_t>(n_split) * B * n_new * H_q * sizeof(float);
  return (n + 255) & ~size_t(255);
}

size_t decode_workspace_bytes(int B, int n_new, int H_q, int H_kv, int d, int L_max) {
  const DecodePlan pl = decode_plan(B, H_q, H_kv, L_max);
  if (pl.n_split <= 1) return 0;
  return decode_part_l_bytes(pl.n_split, B, n_new, H_q) +
         static_cast<size_t>(pl.n_split) * B * n_new * H_q * d * sizeof(float);
}

template <int D>
sqa_status_t launch_decode(const void* q, const void* kc, const void* vc, const int* lens, void* out, int out_bf16,
                           float* lse, int B, int n_new, int H_q, int H_kv, int L_max, float scale, void* ws,
                           cudaStream_t st) {
  using C = sqa::DecCfg<D>;
  const DecodePlan pl = decode_plan(B, H_q, H_kv, L_max);
  if (pl.g * n_new > 128) return SQA_ERR_UNSUPPORTED;  // one 128-row query tile per CTA
  if (static_cast<size_t>(B) * n_new * H_q > 0x7fffffffu) return SQA_ERR_UNSUPPORTED;  // one combine block per row
  CUtensorMap mq, mk, mv;
  const CUtensorMapSwizzle swz = tma_swizzle_for_row_bytes(C::kRowBytes);
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(H_q), uint64_t(n_new), uint64_t(B)};
    const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(H_q) * D * 2, uint64_t(n_new) * H_q * D * 2};
    const uint32_t box[4] = {uint32_t(C::kRowElems), uint32_t(pl.g), uint32_t(n_new), 1};
    if (!make_map_bf16(&mq, q, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(H_kv), uint64_t(L_max), uint64_t(B)};
    const uint64_t strides[3] = {uint64_t(D) * 2, uint64_t(H_kv) * D * 2, uint64_t(L_max) * H_kv * D * 2};
    const uint32_t box[4] = {uint32_t(C::kRowElems), 1, uint32_t(C::kBK), 1};
    if (!make_map_bf16(&mk, kc, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
    if (!make_map_bf16(&mv, vc, 4, dims, strides, box, swz)) return SQA_ERR_CUDA;
  }
  sqa::DecParams p;
  p.out = out;
  p.lse = lse;
  p.part_l = pl.n_split > 1 ? static_cast<float*>(ws) : nullptr;
  p.part_o = pl.n_split > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                                       decode_part_l_bytes(pl.n_split, B, n_new, H_q))
                            : nullptr;
  p.cache_lens = lens;
  p.B = B;
  p.n_new = n_new;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.G = H_q / H_kv;
  p.g = pl.g;
  p.log2g = pl.log2g;
  p.n_sub = pl.n_sub;
  p.L_max = L_max;
  p.chunk = pl.chunk;
  p.n_split = pl.n_split;
  p.out_bf16 = out_bf16;
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long gy = static_cast<long long>(H_kv) * pl.n_sub;
  if (gy > 65535 || B > 65535) return SQA_ERR_UNSUPPORTED;
  auto kern = sqa::sqa_decode_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return SQA_ERR_CUDA;
  dim3 grid(pl.n_split, static_cast<unsigned>(gy), B);
  const sqa_status_t s = launch_k(kern, grid, dim3(sqa::kDecThreads), C::kSmemBytes, st, mq, mk, mv, p);
  if (s != SQA_OK) return s;
  if (pl.n_split > 1) {
    const size_t rows = static_cast<size_t>(B) * n_new * H_q;
    // Its launch overlaps the decode grid's last CTAs (which signal once
    // their last load is issued).
    return launch_k(sqa::decode_combine_kernel<D>, dim3(static_cast<unsigned>(rows)), dim3(sqa::kCombineWarps * 32),
                    0, st, p);
  }
  return launch_status();
}

// Byte offset of head `h` within one token row of d-element heads.
inline const void* head_ptr(const void* base, int h, int d, size_t elem) {
  return base ? static_cast<const uint8_t*>(base) + static_cast<size_t>(h) * d * elem : nullptr;
}
inline void* head_ptr(void* base, int h, int d, size_t elem) {
  return base ? static_cast<uint8_t*>(base) + static_cast<size_t>(h) * d * elem : nullptr;
}

}  // namespace

extern "C" {

sqa_status_t sqa_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H_q, int H_kv,
                          int d_head, int causal, float scale, void* stream) {
  return attn_fwd_impl(q, k, v, out, SQA_DT_F32, nullptr, dense_desc(B, N, N, H_q, H_kv, d_head, causal, scale),
                       stream);
}

sqa_status_t sqa_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, sqa_dtype_t out_dtype,
                             float* lse, int B, int N, int H_q, int H_kv, int d_head, int causal, float scale,
                             void* stream) {
  return attn_fwd_impl(q, k, v, out, out_dtype, lse, dense_desc(B, N, N, H_q, H_kv, d_head, causal, scale), stream);
}

sqa_status_t sqa_attn_fwd_cross(const void* q, const void* k, const void* v, void* out, sqa_dtype_t out_dtype,
                                float* lse, int B, int N_q, int N_kv, int H_q, int H_kv, int d_head, float scale,
                                void* stream) {
  return attn_fwd_impl(q, k, v, out, out_dtype, lse, dense_desc(B, N_q, N_kv, H_q, H_kv, d_head, 0, scale),
                       stream);
}

sqa_status_t sqa_attn_fwd_window(const void* q, const void* k, const void* v, void* out, sqa_dtype_t out_dtype,
                                 float* lse, int B, int N, int H_q, int H_kv, int d_head, int window_left,
                                 int window_right, float scale, void* stream) {
  return attn_fwd_impl(q, k, v, out, out_dtype, lse,
                       window_desc(B, N, H_q, H_kv, d_head, window_left, window_right, scale), stream);
}

size_t sqa_attn_decode_workspace_size(int B, int n_new, int H_q, int H_kv, int d_head, int L_max) {
  if (B <= 0 || n_new <= 0 || H_q <= 0 || H_kv <= 0 || H_kv > H_q || H_q % H_kv != 0 || d_head <= 0 ||
      L_max < n_new)
    return 0;
  return decode_workspace_bytes(B, n_new, H_q, H_kv, d_head, L_max);
}

sqa_status_t sqa_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* cache_lens,
                             void* out, sqa_dtype_t out_dtype, float* lse, int B, int n_new, int H_q, int H_kv,
                             int d_head, int L_max, float scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
  sqa_status_t s = check_attn_args(q, k_cache, v_cache, B, n_new, H_q, H_kv, d_head, scale);
  if (s != SQA_OK) return s;
  if (!cache_lens || !out || L_max < n_new) return SQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cache_lens) & 3u) != 0 || !aligned16(out) || (lse && !aligned16(lse)))
    return SQA_ERR_INVALID_ARG;
  if (out_dtype != SQA_DT_F32 && out_dtype != SQA_DT_BF16) return SQA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * L_max * H_kv > (1ll << 31) - 1) return SQA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, n_new, H_q, H_kv, d_head, L_max);
  if (need > 0 && (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need))
    return SQA_ERR_INVALID_ARG;
  const int ob = out_dtype == SQA_DT_BF16;
  cudaStream_t st = as_stream(stream);
  switch (d_head) {
    case 16:
      return launch_decode<16>(q, k_cache, v_cache, cache_lens, out, ob, lse, B, n_new, H_q, H_kv, L_max, scale,
                               workspace, st);
    case 32:
      return launch_decode<32>(q, k_cache, v_cache, cache_lens, out, ob, lse, B, n_new, H_q, H_kv, L_max, scale,
                               workspace, st);
    case 64:
      return launch_decode<64>(q, k_cache, v_cache, cache_lens, out, ob, lse, B, n_new, H_q, H_kv, L_max, scale,
                               workspace, st);
    default:
      return launch_decode<128>(q, k_cache, v_cache, cache_lens, out, ob, lse, B, n_new, H_q, H_kv, L_max, scale,
                                workspace, st);
  }
}

sqa_status_t sqa_attn_fwd_packed(const void* qkv, void* out, sqa_dtype_t out_dtype, float* lse, int B, int N,
                                 int H_q, int H_kv, int d_head, int causal, float scale, void* stream) {
  if (H_q <= 0 || H_kv <= 0 || d_head <= 0 || H_q > (1 << 20) || H_kv > (1 << 20)) return SQA_ERR_INVALID_ARG;
  return attn_fwd_impl(qkv, head_ptr(qkv, H_q, d_head, 2), head_ptr(qkv, H_q + H_kv, d_head, 2), out, out_dtype,
                       lse, packed_desc(B, N, H_q, H_kv, d_head, causal, scale), stream);
}

size_t sqa_attn_bwd_workspace_size(int B, int N, int H_q, int H_kv, int d_head) {
  if (B <= 0 || N <= 0 || H_q <= 0 || H_kv <= 0 || H_kv > H_q || H_q % H_kv != 0 || d_head <= 0) return 0;
  return bwd_workspace_bytes(B, N, H_q);
}

sqa_status_t sqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, sqa_dtype_t o_dtype,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                          int B, int N, int H_q, int H_kv, int d_head, int causal, float scale, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return attn_bwd_impl(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype,
                       dense_desc(B, N, N, H_q, H_kv, d_head, causal, scale), workspace, workspace_bytes, stream);
}

sqa_status_t sqa_attn_bwd_cross(const void* q, const void* k, const void* v, const void* out, sqa_dtype_t o_dtype,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                sqa_dtype_t grad_dtype, int B, int N_q, int N_kv, int H_q, int H_kv, int d_head,
                                float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return attn_bwd_impl(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype,
                       dense_desc(B, N_q, N_kv, H_q, H_kv, d_head, 0, scale), workspace, workspace_bytes, stream);
}

sqa_status_t sqa_attn_bwd_window(const void* q, const void* k, const void* v, const void* out, sqa_dtype_t o_dtype,
                                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                 sqa_dtype_t grad_dtype, int B, int N, int H_q, int H_kv, int d_head,
                                 int window_left, int window_right, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return attn_bwd_impl(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype,
                       window_desc(B, N, H_q, H_kv, d_head, window_left, window_right, scale), workspace,
                       workspace_bytes, stream);
}

sqa_status_t sqa_attn_bwd_packed(const void* qkv, const void* out, sqa_dtype_t o_dtype, const void* dout,
                                 const float* lse, void* dqkv, sqa_dtype_t grad_dtype, int B, int N, int H_q,
                                 int H_kv, int d_head, int causal, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (H_q <= 0 || H_kv <= 0 || d_head <= 0 || H_q > (1 << 20) || H_kv > (1 << 20)) return SQA_ERR_INVALID_ARG;
  if (grad_dtype != SQA_DT_F32 && grad_dtype != SQA_DT_BF16) return SQA_ERR_INVALID_ARG;
  const size_t ge = grad_dtype == SQA_DT_BF16 ? 2 : 4;
  return attn_bwd_impl(qkv, head_ptr(qkv, H_q, d_head, 2), head_ptr(qkv, H_q + H_kv, d_head, 2), out, o_dtype,
                       dout, lse, dqkv, head_ptr(dqkv, H_q, d_head, ge), head_ptr(dqkv, H_q + H_kv, d_head, ge),
                       grad_dtype, packed_desc(B, N, H_q, H_kv, d_head, causal, scale), workspace, workspace_bytes,
                       stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without a caller workspace: the scratch is this file-scope device
// array, present on every GPU that loads the library until the process exits.
// In host code `g_bwd_static_scratch` names a host-side shadow, never the
// device memory: its device address comes from cudaGetSymbolAddress, looked
// up with the device current, once per device and context.  A device reset
// (cudaDeviceReset) destroys the context and with it the module's memory;
// the next call sees a new context ID and looks the address up again.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_bwd_static_scratch[SQA_BWD_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};
unsigned long long g_static_scratch_ctx[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_fn_once;

// Unique ID of the calling thread's current context, 0 if unknown.
unsigned long long current_context_id() {
  std::call_once(g_ctx_fn_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current == nullptr || g_ctx_id == nullptr || g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      g_ctx_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array in the current device's context, or
// null.  Looked up again whenever the context differs from the one the
// cached address belongs to (or when the context cannot be identified).
void* static_scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (g_static_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_static_scratch_ctx[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_static_scratch) != cudaSuccess) return nullptr;
    g_static_scratch_addr[dev] = ptr;
    g_static_scratch_ctx[dev] = current_context_id();  // the lookup makes the primary context current
  }
  return g_static_scratch_addr[dev];
}
}  // namespace

extern "C" {

sqa_status_t sqa_attn_bwd_static(const void* q, const void* k, const void* v, const void* out, sqa_dtype_t o_dtype,
                                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                 sqa_dtype_t grad_dtype, int B, int N, int H_q, int H_kv, int d_head, int causal,
                                 float scale, void* stream) {
  const size_t need = sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head);
  if (need == 0) return SQA_ERR_INVALID_ARG;
  if (need > SQA_BWD_STATIC_SCRATCH_BYTES) return SQA_ERR_UNSUPPORTED;
  void* scratch = static_scratch_on_current_device();
  if (scratch == nullptr) return SQA_ERR_CUDA;
  return sqa_attn_bwd(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv, d_head, causal,
                      scale, scratch, SQA_BWD_STATIC_SCRATCH_BYTES, stream);
}

sqa_status_t sqa_proj(const void* x, const void* w, const float* bias, void* y, sqa_dtype_t y_dtype, int M, int K,
                      int Nout, void* stream) {
  return gemm_impl(x, false, w, false, bias, y, y_dtype, 0, M, Nout, K, stream);
}

sqa_status_t sqa_gemm(const void* a, sqa_layout_t a_layout, const void* b, sqa_layout_t b_layout, const float* bias,
                      void* c, sqa_dtype_t c_dtype, int accumulate, int M, int N, int K, void* stream) {
  if ((a_layout != SQA_K_CONTIGUOUS && a_layout != SQA_MN_CONTIGUOUS) ||
      (b_layout != SQA_K_CONTIGUOUS && b_layout != SQA_MN_CONTIGUOUS))
    return SQA_ERR_INVALID_ARG;
  return gemm_impl(a, a_layout == SQA_MN_CONTIGUOUS, b, b_layout == SQA_MN_CONTIGUOUS, bias, c, c_dtype,
                   accumulate ? 1 : 0, M, N, K, stream);
}

sqa_status_t sqa_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SQA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, sqa::g_status_word, sizeof(word)) != cudaSuccess) return SQA_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(sqa::g_status_word, &zero, sizeof(zero)) != cudaSuccess) return SQA_ERR_CUDA;
    // A timed-out wait outranks a clamped decode length.
    return (word & sqa::kStatusTimeout) ? SQA_ERR_TIMEOUT : SQA_ERR_INVALID_ARG;
  }
  return SQA_OK;
}

sqa_status_t sqa_selftest_wait_timeout(int timeout_ms, void* stream) {
  if (timeout_ms < 1 || timeout_ms > 10000) return SQA_ERR_INVALID_ARG;
  sqa::selftest_wait_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(timeout_ms) * 1000000ull);
  return launch_status();
}

const char* sqa_status_string(sqa_status_t status) {
  switch (status) {
    case SQA_OK: return "SQA_OK";
    case SQA_ERR_INVALID_ARG: return "SQA_ERR_INVALID_ARG";
    case SQA_ERR_UNSUPPORTED: return "SQA_ERR_UNSUPPORTED";
    case SQA_ERR_CUDA: return "SQA_ERR_CUDA";
    case SQA_ERR_TIMEOUT: return "SQA_ERR_TIMEOUT";
  }
  return "SQA_ERR_UNKNOWN";
}

const char* sqa_version(void) { return "0.3.0"; }

}  // extern "C"
