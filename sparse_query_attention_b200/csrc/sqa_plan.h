// sqa_plan.h - the launch plans of the library as pure host functions: from
// a problem's shape and a few facts about the device (SM count, how many
// thread-block clusters of a size run at once) to tile packing, raster,
// grid and split choices.  No CUDA call is made here, so the plans are
// compiled and checked on the CPU as they are (tests/test_plan.py) and used
// by sqa_api.cu with the device's facts.
#pragma once

#include <algorithm>

namespace sqa {
namespace plan {

// Packing factor of the attention tiles: the largest power of two dividing
// G = H_q / H_kv, at most 128 (query heads of one KV group per 128-row tile).
inline int head_pack(int G) {
  int g = 1;
  while (g < 128 && (G % (2 * g)) == 0) g *= 2;
  return g;
}

// Raster of the persistent GEMMs (row tiles per group of the tile walk):
// the smaller operand stays resident in L2 while the other streams through
// once.  kResident leaves most of the 126 MB L2 (two halves, one per die) to
// the streamed operand's tiles in flight and to the output.
inline int gemm_group_m(int M, int N, int K, int bm) {
  constexpr long long kResident = 40ll << 20;
  const long long a_bytes = 2ll * M * K;
  const long long b_bytes = 2ll * N * K;
  if (b_bytes <= kResident && b_bytes <= a_bytes) return 1;  // N fastest: B stays
  if (a_bytes <= kResident) return (M + bm - 1) / bm;        // M fastest: A stays
  return 8;  // both large: groups of 8 row tiles share each pass over B
}

// KV-cache decode chunking: at least two waves of two CTAs per SM over the
// (batch, key/value head, head sub-group) units, chunks of at least 256 keys
// and a multiple of the 64-key step; among split counts up to four times
// that minimum, the smallest whose last wave is at least 95 % full (else the
// fullest).  Fewer, longer chunks (one wave at most) measured 1-6 % faster
// on a cool GPU but 2-25 % slower after seconds of tensor work at the power
// cap.  Depends only on the shape, so the workspace size is known before the
// lengths are.
constexpr int kDecodeSMs = 148;
constexpr int kDecodeSlots = 2 * kDecodeSMs;  // CTAs resident at once

struct DecodePlan {
  int g, log2g, n_sub, chunk, n_split;
};

inline DecodePlan decode_plan(int B, int H_q, int H_kv, int L_max) {
  DecodePlan pl;
  const int G = H_q / H_kv;
  pl.g = head_pack(G);
  pl.log2g = 0;
  while ((1 << pl.log2g) < pl.g) ++pl.log2g;
  pl.n_sub = G / pl.g;
  const long long units = static_cast<long long>(B) * H_kv * pl.n_sub;
  const long long max_split = (L_max + 255) / 256 > 0 ? (L_max + 255) / 256 : 1;
  const long long n_min = std::min(max_split, std::max(1LL, (2LL * kDecodeSlots + units - 1) / units));
  const long long n_max = std::min(max_split, 4 * n_min);
  long long n = n_min;
  double best = -1.0;
  for (long long c = n_min; c <= n_max; ++c) {
    const long long ctas = units * c;
    const double fill = static_cast<double>(ctas) / (((ctas + kDecodeSlots - 1) / kDecodeSlots) * kDecodeSlots);
    if (fill >= 0.95) {
      n = c;
      break;
    }
    if (fill > best) {
      best = fill;
      n = c;
    }
  }
  const long long per = (L_max + n - 1) / n;
  pl.chunk = static_cast<int>((per + 63) / 64 * 64);
  pl.n_split = static_cast<int>((L_max + pl.chunk - 1) / pl.chunk);
  return pl;
}

// Cover of an unmasked d = 128 forward by its wave counts on `sms` SMs (one
// CTA per SM): the two-tile grid (n_tblk token blocks, two query tiles per
// CTA), the split grid (n_tiles query tiles, one per CTA, each CTA's work
// halved at a rate measured ~8 % lower: a split wave costs kSplitWave of a
// two-tile wave), or both: the two-tile kernel on the n_a token blocks whose
// CTAs fill whole waves, then the split kernel on the remaining
// n_tiles - 2 n_a tiles.  `yz` is the CTA count per token block (KV heads x
// head sub-groups x batch).  Masked problems keep the two-tile grid: the
// longest-first order already packs their waves.
enum class FwdCover { kTwoTile, kSplit, kMixed };

struct FwdWavePlan {
  FwdCover cover;
  int n_a;  // token blocks of the two-tile launch (kMixed)
};

inline FwdWavePlan fwd_wave_plan(long long n_tblk, long long yz, long long n_tiles, int sms, bool masked) {
  constexpr double kSplitWave = 0.55;
  FwdWavePlan r{FwdCover::kTwoTile, 0};
  if (masked || sms <= 0 || yz <= 0) return r;
  auto waves = [&](long long ctas) { return static_cast<double>((ctas + sms - 1) / sms); };
  const double t_two = waves(n_tblk * yz);
  const double t_split = kSplitWave * waves(n_tiles * yz);
  const int n_a = static_cast<int>((n_tblk * yz / sms) * sms / yz);
  const double t_mix = n_a > 0 && n_a < n_tblk ? waves(static_cast<long long>(n_a) * yz) +
                                                    kSplitWave * waves((n_tiles - 2LL * n_a) * yz)
                                              : 1e30;
  if (t_split < 0.97 * t_two && t_split <= t_mix) return {FwdCover::kSplit, 0};
  if (t_mix < 0.97 * t_two) return {FwdCover::kMixed, n_a};
  return r;
}

// Split of a long reduction over a thread-block cluster (split-K GEMM, the
// key range of the forward and of dQ, the query steps of dK/dV): the largest
// cluster size c in max_split, max_split / 2, ..., 2 (powers of two) for
// which each CTA keeps at least `min_work` of the `work` steps and all
// `units` clusters run at once (units <= max_clusters(c), the device's
// count); 1 when none qualifies.
template <typename MaxClusters>
int cluster_split(long long units, long long work, long long min_work, int max_split, MaxClusters max_clusters) {
  for (int c = max_split; c >= 2; c /= 2) {
    if (work < min_work * c) continue;
    if (units <= static_cast<long long>(max_clusters(c))) return c;
  }
  return 1;
}

}  // namespace plan
}  // namespace sqa
