// plan_harness.cpp - C entry points over the library's launch plans
// (sparse_query_attention_b200/csrc/sqa_plan.h) for tests/test_plan.py, which
// compiles this file with g++ (no CUDA) and calls it through ctypes.
#include "sqa_plan.h"

extern "C" {

int h_head_pack(int G) { return sqa::plan::head_pack(G); }

int h_gemm_group_m(int M, int N, int K, int bm) { return sqa::plan::gemm_group_m(M, N, K, bm); }

// out: g, log2g, n_sub, chunk, n_split
void h_decode_plan(int B, int H_q, int H_kv, int L_max, int* out) {
  const sqa::plan::DecodePlan p = sqa::plan::decode_plan(B, H_q, H_kv, L_max);
  out[0] = p.g;
  out[1] = p.log2g;
  out[2] = p.n_sub;
  out[3] = p.chunk;
  out[4] = p.n_split;
}

int h_decode_slots() { return sqa::plan::kDecodeSlots; }

// out: cover (0 two-tile, 1 split, 2 mixed), n_a
void h_fwd_wave_plan(long long n_tblk, long long yz, long long n_tiles, int sms, int masked, int* out) {
  const sqa::plan::FwdWavePlan p = sqa::plan::fwd_wave_plan(n_tblk, yz, n_tiles, sms, masked != 0);
  out[0] = static_cast<int>(p.cover);
  out[1] = p.n_a;
}

// max_clusters[l]: clusters of 2^l CTAs the device runs at once (l = 0..4)
int h_cluster_split(long long units, long long work, long long min_work, int max_split, const int* max_clusters) {
  return sqa::plan::cluster_split(units, work, min_work, max_split, [&](int c) {
    int l = 0;
    while ((1 << l) < c) ++l;
    return max_clusters[l];
  });
}

}  // extern "C"
