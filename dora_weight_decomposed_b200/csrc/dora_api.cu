// C ABI of the DoRA layer library: argument checks, workspace planning and
// dispatch to the bf16 (tcgen05) or fp32 (SIMT) implementation. No call
// allocates device memory or synchronises (except dora_device_status).
#include <cmath>
#include <cstring>
#include <string>

#include "dora_internal.h"

namespace dora {

static thread_local std::string t_last_error;

void set_error(const std::string& msg) { t_last_error = msg; }

int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;  // no device visible: plan for a full B200
  }
  return sms;
}

static inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
static inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Pick how many K splits a GEMM gets. Model (in units of one k-block's
// main-loop time on one SM, kb_bytes of operands): each CTA costs its
// k-blocks + 4 (prologue, TMEM, tails) + its output tile traffic (bf16 when
// not split, fp32 partials when split); CTAs run in waves of one per SM; a
// split GEMM adds a reduction pass over all partials (write + read).
static Split choose_split(int64_t tiles, int64_t kb, int sms, double kb_bytes, double tile_out_elems,
                          double out_elems, int64_t max_splits = 64) {
  Split best;
  best.splits = 1;
  best.kb_per_split = (int)std::max<int64_t>(kb, 1);
  if (kb <= 1 || tiles <= 0) return best;
  double best_t = 1e300;
  for (int64_t n = 1; n <= std::min<int64_t>(kb, std::max<int64_t>(max_splits, 1)); ++n) {
    const int64_t kps = cdiv(kb, n);
    const int64_t ns = cdiv(kb, kps);
    const int64_t waves = cdiv(tiles * ns, sms);
    const double tile_out = tile_out_elems * (ns > 1 ? 4.0 : 2.0) / kb_bytes;
    const double reduce = ns > 1 ? (double)ns * out_elems * 8.0 / ((double)sms * kb_bytes) : 0.0;
    const double t = (double)waves * ((double)kps + 4.0 + tile_out) + reduce;
    if (t < best_t - 1e-9) {
      best_t = t;
      best.splits = (int)ns;
      best.kb_per_split = (int)kps;
    }
  }
  return best;
}

// Tile width and K split of a narrow GEMM (M x N with N = r, long K) on CTA
// pairs (256-row tiles), by a time model in microseconds at ~1.9 GHz:
//  - a k-block takes the longer of its MMAs (2 clocks per tile column) and
//    bringing each CTA's (128 + bn/2) x 128 operand bytes in (~58 bytes per
//    clock per SM, the TMA rate the main loops sustain);
//  - the epilogue stores a 128 x bn tile per CTA: bf16 directly (~17 GB/s per
//    SM) or, when K is split, fp32 partials by TMA (~100 GB/s per SM);
//  - each wave of pairs (one per two SMs) adds a fixed 2 us;
//  - a split K loop adds the reduction pass over all partials (~4.5 TB/s)
//    and its launch (4 us).
struct NarrowChoice {
  int bn = 128;
  Split split;
  bool pair = true;
};

// The same on single CTAs (128-row tiles, operand bytes (128 + bn) x 128 per
// k-block), which measured faster for dB and dA (K = T, both operands
// token-major): 128 x 192 tiles there keep every SM busy without a K split.
static NarrowChoice choose_narrow_1cta(int64_t M, int64_t N, int64_t K, bool b_mn, int sms) {
  static const int kCandK[] = {16, 32, 64, 128, 192, 256, 384, 512};
  static const int kCandMN[] = {64, 128, 192, 256, 384, 512};
  const int* cand = b_mn ? kCandMN : kCandK;
  const int ncand = b_mn ? 6 : 8;
  const int64_t kb = std::max<int64_t>(cdiv(K, 64), 1);
  NarrowChoice best;
  best.pair = false;
  double best_t = 1e300;
  for (int ci = 0; ci < ncand; ++ci) {
    const int bn = cand[ci];
    if (ci > 0 && cand[ci - 1] >= N) break;
    const int64_t tiles = cdiv(M, 128) * cdiv(N, bn);
    const double kb_clk = std::max(2.0 * bn, (128.0 + bn) * 1.28);
    for (int64_t ns = 1; ns <= std::min<int64_t>(kb, 32); ++ns) {
      const int64_t kps = cdiv(kb, ns);
      const int64_t splits = cdiv(kb, kps);
      if (splits != ns) continue;
      const int64_t waves = cdiv(tiles * splits, sms);
      double t = (double)waves * ((double)kps * kb_clk / 1900.0 + 2.0);
      if (splits > 1) t += (double)splits * M * N * 8.0 / 3.0e6 + 4.0;
      if (t < best_t - 1e-9) {
        best_t = t;
        best.bn = bn;
        best.split.splits = (int)splits;
        best.split.kb_per_split = (int)kps;
      }
    }
  }
  return best;
}

// Tile width and pairs per cluster (K splits reduced in the cluster) of a narrow
// GEMM on CTA-pair clusters: the narrowest pair tile that covers N, and of 1 to
// 4 pairs per cluster the one with the least estimated time, in units of one
// k-block's main-loop time: waves of clusters (as many at once as the device
// holds: a cluster must fit in one GPC) times the k-blocks of a split, plus a
// fixed cost per tile (prologue, pipeline fill, drain, stores) and per extra
// split of the reduction. Ties go to fewer splits.
struct ClusterChoice {
  int bn = 128;
  int cs = 1;
};

// Clusters of cs pairs resident at once: the device's answer, else SMs / (2 cs)
// less one GPC's worth for clusters above two pairs.
static int64_t resident_clusters(int cs, int sms) {
  const int n = max_active_pair_clusters(cs);
  if (n > 0) return n;
  const int64_t even = std::max(1, sms / (2 * cs));
  return cs > 2 ? std::max<int64_t>(1, even - 3) : even;
}

static ClusterChoice choose_narrow_cluster_bn(int64_t M, int64_t N, int64_t K, int bn, int sms);

// The rank may also be split into two column tiles: 192 of r = 384 or 128 of r = 256 with
// B read K-major; with B read MN-major (whole 64-column chunks per CTA) 256 and a
// half-empty second tile for r = 384. Twice the tiles to spread over the SM pairs at the
// same k-block count, for twice the reads of the A operand (from L2) per column. Chosen
// when the time model (microseconds, as for the base GEMMs below) says so.
static ClusterChoice choose_narrow_cluster(int64_t M, int64_t N, int64_t K, bool b_mn, int sms) {
  const int full = b_mn ? (N <= 128 ? 128 : N <= 256 ? 256 : N <= 384 ? 384 : 512) : (int)bn_pair_k(N);
  ClusterChoice c = choose_narrow_cluster_bn(M, N, K, full, sms);
  const int half = N > 256 && N <= 384 ? (b_mn ? 256 : 192) : (!b_mn && N > 128 && N <= 256) ? 128 : 0;
  if (half == 0) return c;
  const int64_t kb = std::max<int64_t>(cdiv(K, 64), 1);
  auto us = [&](const ClusterChoice& x) {
    const double kb_us = std::max(2.0 * 256.0 * x.bn * 64.0 / 23.0e6, (16384.0 + 64.0 * x.bn) / 110.0e3);
    const int64_t tiles = cdiv(M, 256) * cdiv(N, x.bn);
    return (double)cdiv(tiles, resident_clusters(x.cs, sms)) * ((double)cdiv(kb, x.cs) * kb_us + 1.5) +
           0.75 * (x.cs - 1) * x.bn / 128.0 + 1.0;
  };
  const ClusterChoice h = choose_narrow_cluster_bn(M, N, K, half, sms);
  return us(h) < us(c) ? h : c;
}

static ClusterChoice choose_narrow_cluster_bn(int64_t M, int64_t N, int64_t K, int bn, int sms) {
  ClusterChoice c;
  c.bn = bn;
  const int64_t tiles = cdiv(M, 256) * cdiv(N, c.bn);
  const int64_t kb = std::max<int64_t>(cdiv(K, 64), 1);
  double best = 1e300;
  // Clusters of 8 pairs (16 CTAs, a non-portable size) for tiles up to 128 columns wide,
  // when the device reports that it can hold them.
  const bool eight = bn <= 128 && max_active_pair_clusters(8) > 0;
  for (int cs : {1, 2, 3, 4, 8}) {
    if (cs == 8 && !eight) break;
    if (cs > 1 && kb < 2 * cs) break;  // at least two k-blocks per split
    const int64_t waves = cdiv(tiles, resident_clusters(cs, sms));
    const double t = (double)waves * ((double)cdiv(kb, cs) + 4.0) + (cs > 1 ? 1.0 * (cs - 1) * c.bn / 128.0 : 0.0);
    if (t < best - 1e-9) {
      best = t;
      c.cs = cs;
    }
  }
  return c;
}

// The 256 x 256 base GEMMs (forward, dx): the persistent pair kernel (0) or clusters of
// 1 to 4 pairs (the cluster kernel; with more than one pair per cluster the pairs split K).
// Estimated microseconds at ~1.9 GHz: a pair k-block takes the longer of its MMAs and its
// operand loads (~110 GB/s per SM); each wave adds 1.5 us (prologue, pipeline fill), each
// extra split 1.5 us of reduction, and a cluster launch 1 us for its stores. The persistent
// kernel overlaps each tile's epilogue with the next tile's main loop, so only its waves count,
// except in a single wave of one tile per pair: nothing hides that epilogue's row-per-thread
// stores (~8 us for the forward's two outputs), where the cluster kernel stores from shared
// memory (c4b forward: 48 tiles of 33 k-blocks took 33.4 us persistent under ncu, the c4a
// forward's 3-pair clusters with the same k-blocks per pair 23.2 us). (256 x 128 cluster
// tiles, twice as many, measured slower: 25.2 against 22.6 us for the c4a forward.)
static int choose_wide_cs(int64_t M, int64_t N, int64_t K, int sms) {
  const int64_t tiles = cdiv(M, 256) * cdiv(N, 256);
  const int64_t kb = std::max<int64_t>(cdiv(K, 64), 1);
  const int pairs = std::max(1, sms / 2);
  const double kb_us = std::max(2.0 * 256.0 * 256.0 * 64.0 / 23.0e6, (16384.0 + 64.0 * 256.0) / 110.0e3);
  const int64_t waves = cdiv(tiles, pairs);
  double best = (double)waves * ((double)kb * kb_us + 1.5) + (waves == 1 ? 8.0 : 0.0);
  int cs = 0;
  for (int c : {1, 2, 3, 4}) {
    if (c > 1 && kb < 2 * c) break;
    const int64_t rc = resident_clusters(c, sms);
    if (c == 1 && tiles > rc) continue;  // one pair per tile only in a single wave
    const double t = (double)cdiv(tiles, rc) * ((double)cdiv(kb, c) * kb_us + 1.5) + 1.5 * (c - 1) + 1.0;
    if (t < best - 1e-9) {
      best = t;
      cs = c;
    }
  }
  return cs;
}

// dB and dA (both K = T, tile width bn) in one grouped persistent launch of whole
// tiles, or as two cluster split-K launches: estimated microseconds at ~1.9 GHz,
// a pair k-block taking the longer of its MMAs and its operand loads (~110 GB/s
// per SM); a fixed 4 us for the grouped launch and 10 us per cluster launch
// (prologue, accumulator drain, cluster reduction, stores).
static bool dBA_grouped(int64_t d_out, int64_t d_in, int64_t r, int64_t T, int bn, int sms) {
  const int64_t kb = std::max<int64_t>(cdiv(T, 64), 1);
  const int pairs = std::max(1, sms / 2);
  const double kb_us = std::max(2.0 * 256.0 * bn * 64.0 / 23.0e6, (16384.0 + 64.0 * bn) / 110.0e3);
  const int64_t tB = cdiv(d_out, 256) * cdiv(r, bn), tA = cdiv(d_in, 256) * cdiv(r, bn);
  const double grouped = (double)cdiv(tB + tA, pairs) * (double)kb * kb_us + 4.0;
  auto clustered = [&](int64_t tiles) {
    double best = 1e300;
    for (int cs : {1, 2, 3, 4}) {
      if (cs > 1 && kb < 2 * cs) break;
      best = std::min(best, (double)cdiv(tiles, resident_clusters(cs, sms)) * (double)cdiv(kb, cs) * kb_us + 10.0);
    }
    return best;
  };
  return grouped <= clustered(tB) + clustered(tA);
}

// dx and the grouped dB/dA launch read only dz, du and the inputs, and write disjoint
// outputs: both may run at once. When dx's persistent tiles fit on fewer pairs than the
// device has without another wave (or its clusters leave pairs idle), dB/dA takes the
// idle pairs on a second stream, provided its estimate (as in dBA_grouped) stays under
// dx's (as in choose_wide_cs); the step then loses the dB/dA launch from its critical path.
static void plan_backward_fork(Plan& p, int64_t d_out, int64_t d_in, int64_t r, int64_t T) {
  const int pairs = std::max(1, p.sms / 2);
  p.bwd_fork = 0;
  p.dx_defer = 0;
  p.dx_pairs = pairs;
  p.dBA_pairs = pairs;
  if (!p.dBA_grouped) return;
  // pairs the device can place at once (a GPC with an odd SM count strands one SM)
  const int64_t placeable = std::min<int64_t>(pairs, resident_clusters(1, p.sms));
  const int64_t tiles = cdiv(T, 256) * cdiv(d_in, 256);
  const int64_t kb = std::max<int64_t>(cdiv(d_out, 64) + cdiv(r, 64), 1);
  const double kb_us = std::max(2.0 * 256.0 * 256.0 * 64.0 / 23.0e6, (16384.0 + 64.0 * 256.0) / 110.0e3);
  int64_t used;
  double dx_us;
  if (p.dx_cs == 0) {
    const int64_t waves = cdiv(tiles, pairs);
    used = cdiv(tiles, waves);
    dx_us = (double)waves * ((double)kb * kb_us + 1.5);
  } else {
    const int64_t rc = resident_clusters(p.dx_cs, p.sms);
    used = std::min(tiles, rc) * p.dx_cs;
    dx_us = (double)cdiv(tiles, rc) * ((double)cdiv(kb, p.dx_cs) * kb_us + 1.5) + 1.5 * (p.dx_cs - 1) + 1.0;
  }
  const int64_t idle = placeable - used;
  if (idle < 1) return;
  const int bn = p.dB_bn;
  const int64_t kbT = std::max<int64_t>(cdiv(T, 64), 1);
  const double kbT_us = std::max(2.0 * 256.0 * bn * 64.0 / 23.0e6, (16384.0 + 64.0 * bn) / 110.0e3);
  const int64_t tBA = (cdiv(d_out, 256) + cdiv(d_in, 256)) * cdiv(r, bn);
  const double dBA_us = (double)cdiv(tBA, idle) * (double)kbT * kbT_us + 4.0;
  if (dBA_us > dx_us) return;
  p.bwd_fork = 1;
  p.dx_pairs = (int)used;
  p.dBA_pairs = (int)std::min(idle, tBA);
  // dx needs du only for its last k-block ([dz | du] [W0 ; A]): when du's CTAs and dx's fit
  // on the SMs together (one wave each), dx starts beside du, and dB/dA follow their own copy
  // of du on the second stream. That stream then carries du and all of dB/dA, so only where
  // dB/dA take at most two tiles per pair (measured: c4a backward 38.9 -> 32.9 us, c4b
  // 51.2 -> 45.1 us; c3 at T = 256, seven tiles per pair, 141.4 -> 145.5 us).
  const int64_t tiles_du = cdiv(T, 256) * cdiv(r, p.du_bn);
  if (tiles_du <= resident_clusters(p.du_cs, p.sms) && 2 * p.du_cs * tiles_du + 2 * used <= p.sms &&
      cdiv(tBA, p.dBA_pairs) <= 2)
    p.dx_defer = 1;
}

static NarrowChoice choose_narrow(int64_t M, int64_t N, int64_t K, bool b_mn, int sms) {
  static const int kCandK[] = {64, 128, 256, 384, 512};
  static const int kCandMN[] = {128, 256, 384, 512};
  const int* cand = b_mn ? kCandMN : kCandK;
  const int ncand = b_mn ? 4 : 5;
  const int64_t kb = std::max<int64_t>(cdiv(K, 64), 1);
  const int pairs = std::max(1, sms / 2);
  NarrowChoice best;
  double best_t = 1e300;
  for (int ci = 0; ci < ncand; ++ci) {
    const int bn = cand[ci];
    if (ci > 0 && cand[ci - 1] >= N) break;  // wider than needed
    const int64_t tiles = cdiv(M, 256) * cdiv(N, bn);
    const double kb_clk = std::max(2.0 * bn, (128.0 + bn / 2.0) * 128.0 / 58.0);
    for (int64_t ns = 1; ns <= std::min<int64_t>(kb, 32); ++ns) {
      const int64_t kps = cdiv(kb, ns);
      const int64_t splits = cdiv(kb, kps);
      if (splits != ns) continue;
      const int64_t waves = cdiv(tiles * splits, pairs);
      const double epi = splits > 1 ? 128.0 * bn * 4.0 / 1.0e5 : 128.0 * bn * 2.0 / 1.7e4;
      double t = (double)waves * ((double)kps * kb_clk / 1900.0 + epi + 2.0);
      if (splits > 1) t += (double)splits * M * N * 8.0 / 4.5e6 + 4.0;
      if (t < best_t - 1e-9) {
        best_t = t;
        best.bn = bn;
        best.split.splits = (int)splits;
        best.split.kb_per_split = (int)kps;
      }
    }
  }
  return best;
}

Plan make_plan(const dora_desc_t& d, int64_t T, int op) {
  Plan p;
  p.sms = device_sm_count();
  p.fwd_pairs = std::max(1, p.sms / 2);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const int64_t r = d.r, d_in = d.d_in, d_out = d.d_out;
  if (d.dtype == DORA_BF16) {
    const double kbB = 64.0 * 2.0;  // bytes per K element pair of rows (x 64 K per k-block)
    if (op == DORA_OP_NORM) {
      // The Gram kernel (one cluster launch) writes (s/2) G as bf16 hi + lo into
      // off_gs directly. The norm GEMM runs on CTA pairs, 256 rows x the whole
      // rank per tile.
      p.norm_bn = bn_pair_k(r);
      const int64_t norm_tiles = cdiv(d_out, 256), norm_kb = cdiv(d_in, 64) + 2 * cdiv(r, 64);
      p.norm = choose_split(norm_tiles, norm_kb, p.sms / 2, kbB * (128 + p.norm_bn / 2.0), 0.0, (double)d_out);
      if (cdiv(r, 128) == 1 && p.sms / 2 > 8) {
        // A single Gram tile runs beside the norm GEMM on the SMs it leaves (2 to 8 CTAs
        // splitting K), and the norm GEMM's last split waits for it before its final
        // k-blocks. When those SMs are too few for the Gram's K loop to finish within a
        // split's, leave it eight.
        const int64_t spare = p.sms - 2 * std::min<int64_t>(norm_tiles * p.norm.splits, p.sms / 2);
        const int64_t gram_cs = spare >= 8 ? 8 : spare >= 4 ? 4 : 2;
        if (cdiv(cdiv(d_in, 64), gram_cs) > p.norm.kb_per_split)
          p.norm = choose_split(norm_tiles, norm_kb, p.sms / 2 - 4, kbB * (128 + p.norm_bn / 2.0), 0.0,
                                (double)d_out);
      }
      p.off_norm_part = take((size_t)p.norm.splits * d_out * 4);
      p.off_gs = take((size_t)r * 2 * cdiv(r, 64) * 64 * 2);
      // split counters, one per 128-row half of a pair tile, zeroed by the Gram kernel
      p.zero_bytes = (size_t)2 * cdiv(d_out, 256) * 4;
      p.off_ctr = take(p.zero_bytes);
    } else if (op == DORA_OP_FORWARD && T > 0) {
      const ClusterChoice u = choose_narrow_cluster(T, r, d_in, false, p.sms);
      p.u_bn = u.bn;
      p.u_cs = u.cs;
      p.fwd_cs = choose_wide_cs(T, d_out, cdiv(d_in, 64) * 64 + cdiv(r, 64) * 64, p.sms);
      // The base GEMM needs s u only for its last k-block: when its CTAs and u's fit on the
      // SMs together (one wave each), it starts its x W0 main loop beside u.
      {
        const int64_t tiles_u = cdiv(T, 256) * cdiv(r, p.u_bn);
        const int64_t tiles_f = cdiv(T, 256) * cdiv(d_out, 256);
        const int64_t ctas_u = 2 * p.u_cs * tiles_u;
        bool one_wave = tiles_u <= resident_clusters(p.u_cs, p.sms);
        int64_t ctas_f;
        if (p.fwd_cs >= 1) {
          ctas_f = 2 * p.fwd_cs * tiles_f;
          one_wave = one_wave && tiles_f <= resident_clusters(p.fwd_cs, p.sms);
        } else {
          ctas_f = 2 * std::min<int64_t>(tiles_f, std::max(1, p.sms / 2));
        }
        p.fwd_defer = (one_wave && ctas_u + ctas_f <= p.sms) ? 1 : 0;
        // A persistent base GEMM of several waves whose last wave leaves pairs idle runs the
        // same waves on fewer pairs (ceil(tiles / waves)); u then takes the SMs left over, on
        // the largest clusters that fit there, when it is estimated to end before the base
        // GEMM's first tile reaches its s u k-block (c2: 128 tiles in two waves on 64 pairs,
        // u's 8 tiles on 20 SMs).
        const int pairs = std::max(1, p.sms / 2);
        const int64_t waves = cdiv(tiles_f, pairs);
        if (!p.fwd_defer && p.fwd_cs == 0 && waves >= 2) {
          const int64_t fpairs = cdiv(tiles_f, waves);
          const int64_t spare = p.sms - 2 * fpairs;
          const int64_t kb_u = std::max<int64_t>(cdiv(d_in, 64), 1);
          const int64_t kb_f = cdiv(d_in, 64) + cdiv(r, 64);
          const double kbu_us = std::max(2.0 * 256.0 * p.u_bn * 64.0 / 23.0e6, (16384.0 + 64.0 * p.u_bn) / 110.0e3);
          const double kbf_us = std::max(2.0 * 256.0 * 256.0 * 64.0 / 23.0e6, (16384.0 + 64.0 * 256.0) / 110.0e3);
          int cs = 0;
          for (int c : {1, 2, 3, 4})
            if (2 * c * tiles_u <= spare && (c == 1 || kb_u >= 2 * c) && tiles_u <= resident_clusters(c, p.sms)) cs = c;
          if (cs > 0 && (double)cdiv(kb_u, cs) * kbu_us + 3.0 <= (double)kb_f * kbf_us) {
            p.u_cs = cs;
            p.fwd_pairs = (int)fpairs;
            p.fwd_defer = 1;
          }
        }
      }
      p.off_su = take((size_t)T * r * 2);
    } else if ((op == DORA_OP_BACKWARD || op == DORA_OP_BACKWARD_FULL) && T > 0) {
      p.off_dz = take((size_t)T * d_out * 2);
      // Compose backward: 64-column strips x row blocks, sized so that the grid is one
      // wave at five 256-thread blocks per SM (its register use) and no tail is left.
      {
        const int64_t strips = cdiv(d_out, 64), groups = cdiv(T, 32);
        const int64_t per_strip = std::max<int64_t>(1, (int64_t)p.sms * 5 / strips);
        p.dm_rows = (int)(32 * cdiv(groups, std::min(per_strip, groups)));
        p.dm_rowblocks = (int)cdiv(T, p.dm_rows);
      }
      p.off_dm_part = take((size_t)p.dm_rowblocks * d_out * 4);
      const ClusterChoice du = choose_narrow_cluster(T, r, d_out, true, p.sms);
      p.du_bn = du.bn;
      p.du_cs = du.cs;
      p.off_du = take((size_t)T * r * 2);
      p.off_du2 = take((size_t)T * r * 2);  // always, so that the workspace grows with T
      const ClusterChoice dB = choose_narrow_cluster(d_out, r, T, true, p.sms);
      p.dB_bn = dB.bn;
      p.dB_cs = dB.cs;
      const ClusterChoice dA = choose_narrow_cluster(d_in, r, T, true, p.sms);
      p.dA_bn = dA.bn;
      p.dA_cs = dA.cs;
      p.dBA_grouped = dBA_grouped(d_out, d_in, r, T, p.dB_bn, p.sms) ? 1 : 0;
      p.dx_cs = choose_wide_cs(T, d_in, cdiv(d_out, 64) * 64 + cdiv(r, 64) * 64, p.sms);
      plan_backward_fork(p, d_out, d_in, r, T);
      // counters of the dm column strips, zeroed by one memset per call
      p.zero_bytes = (size_t)cdiv(d_out, 64) * 4;
      p.off_ctr = take(p.zero_bytes);
      if (op == DORA_OP_BACKWARD_FULL) {
        const int64_t rp = cdiv(r, 64) * 64;
        p.off_kappa = take((size_t)d_out * 4);
        p.off_bk = take((size_t)d_out * r * 2);
        p.off_gs = take((size_t)r * 2 * rp * 2);
        const NarrowChoice q = choose_narrow(d_out, r, d_in + 2 * rp, false, p.sms);
        p.q_bn = q.bn;
        p.q = q.split;
        p.off_q_part = take((size_t)p.q.splits * d_out * r * 4);
        const NarrowChoice h = choose_narrow_1cta(r, r, d_out, true, p.sms);
        p.h_bn = h.bn;
        p.h = h.split;
        if (p.h.splits > 1) p.off_h_part = take((size_t)p.h.splits * r * r * 4);
        p.off_h = take((size_t)r * r * 2);
      }
    }
  } else {
    if (op == DORA_OP_NORM) {
      p.off_f32_a = take((size_t)d_out * r * 4);
      p.off_f32_b = take((size_t)r * r * 4);
      p.off_f32_c = take((size_t)d_out * r * 4);
    } else if (op == DORA_OP_FORWARD && T > 0) {
      p.off_f32_a = take((size_t)T * r * 4);
      p.off_f32_b = take((size_t)T * d_out * 4);
    } else if ((op == DORA_OP_BACKWARD || op == DORA_OP_BACKWARD_FULL) && T > 0) {
      p.off_f32_a = take((size_t)T * d_out * 4);
      p.off_f32_b = take((size_t)cdiv(T, 64) * d_out * 4);
      p.off_f32_c = take((size_t)T * r * 4);
      if (op == DORA_OP_BACKWARD_FULL) {
        p.off_kappa = take((size_t)d_out * 4);
        p.off_bk = take((size_t)d_out * r * 4);
        p.off_gs = take((size_t)r * r * 4);
        p.off_q_part = take((size_t)d_out * r * 4);
        p.off_h = take((size_t)r * r * 4);
      }
    }
  }
  if (op == DORA_OP_VERA_GRAD) {
    // Row blocks of the dd pass: 64 rows each, at most 296 (two per SM), so the
    // final per-column sum over the blocks stays short.
    p.vera_blocks = (int)std::min<int64_t>(cdiv(d_out, 64), 296);
    p.off_f32_a = take((size_t)p.vera_blocks * r * 4);
  }
  p.total = off;
  return p;
}

// ------------------------------------------------------------------ checks

static const int64_t kMaxDim = (int64_t)65535 * 128;  // grid.y limit on 128-row tiles

static bool check_desc(const dora_desc_t* d) {
  if (!d) return set_error("desc is NULL"), false;
  if (d->dtype != DORA_BF16 && d->dtype != DORA_FP32) return set_error("desc->dtype is not DORA_BF16 or DORA_FP32"), false;
  if (d->d_out < 1 || d->d_in < 1 || d->r < 1) return set_error("d_out, d_in and r must be >= 1"), false;
  if (d->d_out > kMaxDim || d->d_in > kMaxDim) return set_error("d_out or d_in too large"), false;
  if (!std::isfinite(d->s)) return set_error("s is not finite"), false;
  if (d->dtype == DORA_BF16) {
    if (d->d_out % 8 || d->d_in % 8 || d->r % 8)
      return set_error("bf16 layers need d_out, d_in and r to be multiples of 8"), false;
  }
  if (d->r > 512) return set_error("r above 512 is not supported"), false;
  return true;
}

static bool check_T(int64_t T) {
  if (T < 0 || T > kMaxDim) return set_error("T out of range"), false;
  return true;
}

static bool check_ptr(const void* p, const char* name, size_t align) {
  if (!p) return set_error(std::string(name) + " is NULL"), false;
  if (reinterpret_cast<uintptr_t>(p) % align)
    return set_error(std::string(name) + " is not " + std::to_string(align) + "-byte aligned"), false;
  return true;
}

static bool check_opt_ptr(const void* p, const char* name, size_t align) {
  return p == nullptr || check_ptr(p, name, align);
}

static size_t tensor_align(const dora_desc_t* d) { return d->dtype == DORA_BF16 ? 16 : 4; }

// The bf16 path runs tcgen05 kernels built for sm_100a only.
static dora_status_t check_device(const dora_desc_t* d) {
  if (d->dtype != DORA_BF16) return DORA_OK;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    set_error("no CUDA device available");
    return DORA_ECUDA;
  }
  if (major != 10 || minor != 0) {
    set_error("the bf16 path needs an sm_100 (B200) device");
    return DORA_EUNSUPPORTED;
  }
  return DORA_OK;
}

static dora_status_t check_ws(const Plan& p, const void* ws, size_t ws_bytes) {
  if (p.total == 0) return DORA_OK;
  if (!ws) {
    set_error("workspace is NULL but " + std::to_string(p.total) + " bytes are needed");
    return DORA_EWORKSPACE;
  }
  if (reinterpret_cast<uintptr_t>(ws) % 256) {
    set_error("workspace is not 256-byte aligned");
    return DORA_EINVAL;
  }
  if (ws_bytes < p.total) {
    set_error("workspace has " + std::to_string(ws_bytes) + " bytes, needs " + std::to_string(p.total));
    return DORA_EWORKSPACE;
  }
  return DORA_OK;
}

}  // namespace dora

using namespace dora;

extern "C" {

size_t dora_workspace_size(const dora_desc_t* desc, int64_t T, int op) {
  if (!check_desc(desc) || !check_T(T) || op < DORA_OP_NORM || op > DORA_OP_VERA_GRAD) return 0;
  return make_plan(*desc, T, op).total;
}

dora_status_t dora_vera_compose(const dora_desc_t* desc, const void* B_shared, const float* b, const float* d,
                                void* B_out, dora_stream_t stream) {
  if (!check_desc(desc)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  if (!check_ptr(B_shared, "B_shared", al) || !check_ptr(b, "b", 4) || !check_ptr(d, "d", 4) ||
      !check_ptr(B_out, "B_out", al))
    return DORA_EINVAL;
  dora_status_t s = check_device(desc);
  if (s != DORA_OK) return s;
  return vera_compose(*desc, B_shared, b, d, B_out, reinterpret_cast<cudaStream_t>(stream));
}

dora_status_t dora_vera_grad(const dora_desc_t* desc, const void* B_shared, const float* b, const float* d,
                             const void* dB, float* db, float* dd, void* ws, size_t ws_bytes, dora_stream_t stream) {
  if (!check_desc(desc)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  if (!check_ptr(B_shared, "B_shared", al) || !check_ptr(b, "b", 4) || !check_ptr(d, "d", 4) ||
      !check_ptr(dB, "dB", al) || !check_ptr(db, "db", 4) || !check_ptr(dd, "dd", 4))
    return DORA_EINVAL;
  const Plan p = make_plan(*desc, 0, DORA_OP_VERA_GRAD);
  dora_status_t s = check_ws(p, ws, ws_bytes);
  if (s != DORA_OK) return s;
  if ((s = check_device(desc)) != DORA_OK) return s;
  return vera_grad(*desc, p, B_shared, b, d, dB, db, dd, reinterpret_cast<uint8_t*>(ws),
                   reinterpret_cast<cudaStream_t>(stream));
}

dora_status_t dora_merge(const dora_desc_t* desc, const void* W0, const void* A, const void* B, const float* g,
                         void* W_out, void* ws, size_t ws_bytes, dora_stream_t stream) {
  if (!check_desc(desc)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  if (!check_ptr(W0, "W0", al) || !check_ptr(A, "A", al) || !check_ptr(B, "B", al) || !check_ptr(g, "g", 4) ||
      !check_ptr(W_out, "W_out", al))
    return DORA_EINVAL;
  const Plan p = make_plan(*desc, 0, DORA_OP_MERGE);
  dora_status_t s = check_ws(p, ws, ws_bytes);
  if (s != DORA_OK) return s;
  if ((s = check_device(desc)) != DORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (desc->dtype == DORA_BF16) return bf16_merge(*desc, p, W0, A, B, g, W_out, reinterpret_cast<uint8_t*>(ws), st);
  return f32_merge(*desc, (const float*)W0, (const float*)A, (const float*)B, g, (float*)W_out, st);
}

dora_status_t dora_norm(const dora_desc_t* desc, const void* W0, const void* A, const void* B, const float* m,
                        float* norm_out, float* g_out, float* gm1_out, void* ws, size_t ws_bytes,
                        dora_stream_t stream) {
  if (!check_desc(desc)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  if (!check_ptr(W0, "W0", al) || !check_ptr(A, "A", al) || !check_ptr(B, "B", al) || !check_ptr(m, "m", 4) ||
      !check_ptr(norm_out, "norm_out", 4) || !check_ptr(g_out, "g_out", 4) || !check_ptr(gm1_out, "gm1_out", 4))
    return DORA_EINVAL;
  const Plan p = make_plan(*desc, 0, DORA_OP_NORM);
  dora_status_t s = check_ws(p, ws, ws_bytes);
  if (s != DORA_OK) return s;
  if ((s = check_device(desc)) != DORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  if (desc->dtype == DORA_BF16) return bf16_norm(*desc, p, W0, A, B, m, norm_out, g_out, gm1_out, w, st);
  return f32_norm(*desc, p, (const float*)W0, (const float*)A, (const float*)B, m, norm_out, g_out, gm1_out, w, st);
}

dora_status_t dora_forward(const dora_desc_t* desc, int64_t T, const void* x, const void* W0, const void* A,
                           const void* B, const float* gm1, void* y, void* su_save, void* pre_save, void* ws,
                           size_t ws_bytes, dora_stream_t stream) {
  if (!check_desc(desc) || !check_T(T)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  // Per-token tensors have no elements when T == 0 and may then be NULL.
  const bool tok = T > 0;
  if ((tok && !check_ptr(x, "x", al)) || !check_ptr(W0, "W0", al) || !check_ptr(A, "A", al) ||
      !check_ptr(B, "B", al) || !check_ptr(gm1, "gm1", 16) || (tok && !check_ptr(y, "y", al)) ||
      !check_opt_ptr(su_save, "su_save", al) || !check_opt_ptr(pre_save, "pre_save", al))
    return DORA_EINVAL;
  const Plan p = make_plan(*desc, T, DORA_OP_FORWARD);
  dora_status_t s = check_ws(p, ws, ws_bytes);
  if (s != DORA_OK) return s;
  if ((s = check_device(desc)) != DORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  if (desc->dtype == DORA_BF16) return bf16_forward(*desc, p, T, x, W0, A, B, gm1, y, su_save, pre_save, w, st);
  return f32_forward(*desc, p, T, (const float*)x, (const float*)W0, (const float*)A, (const float*)B, gm1,
                     (float*)y, (float*)su_save, (float*)pre_save, w, st);
}

static dora_status_t backward_impl(bool full, const dora_desc_t* desc, int64_t T, const void* dy, const void* x,
                                   const void* W0, const void* A, const void* B, const float* norm, const float* g,
                                   const void* su_save, const void* pre_save, float* dm, void* dA, void* dB,
                                   void* dx, void* ws, size_t ws_bytes, dora_stream_t stream) {
  if (!check_desc(desc) || !check_T(T)) return DORA_EINVAL;
  const size_t al = tensor_align(desc);
  // Per-token tensors have no elements when T == 0 and may then be NULL.
  const bool tok = T > 0;
  if ((tok && !check_ptr(dy, "dy", al)) || (tok && !check_ptr(x, "x", al)) || !check_ptr(W0, "W0", al) ||
      !check_ptr(A, "A", al) || !check_ptr(B, "B", al) || !check_ptr(norm, "norm", 4) || !check_ptr(g, "g", 16) ||
      (tok && !check_ptr(su_save, "su_save", al)) || (tok && !check_ptr(pre_save, "pre_save", al)) ||
      !check_ptr(dm, "dm", 4) || !check_ptr(dA, "dA", al) || !check_ptr(dB, "dB", al) ||
      !check_opt_ptr(dx, "dx", al))
    return DORA_EINVAL;
  const Plan p = make_plan(*desc, T, full ? DORA_OP_BACKWARD_FULL : DORA_OP_BACKWARD);
  dora_status_t s = check_ws(p, ws, ws_bytes);
  if (s != DORA_OK) return s;
  if ((s = check_device(desc)) != DORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  if (desc->dtype == DORA_BF16)
    return (full ? bf16_backward_full : bf16_backward)(*desc, p, T, dy, x, W0, A, B, norm, g, su_save, pre_save, dm,
                                                       dA, dB, dx, w, st);
  return (full ? f32_backward_full : f32_backward)(*desc, p, T, (const float*)dy, (const float*)x, (const float*)W0,
                                                   (const float*)A, (const float*)B, norm, g, (const float*)su_save,
                                                   (const float*)pre_save, dm, (float*)dA, (float*)dB, (float*)dx,
                                                   w, st);
}

dora_status_t dora_backward(const dora_desc_t* desc, int64_t T, const void* dy, const void* x, const void* W0,
                            const void* A, const void* B, const float* norm, const float* g, const void* su_save,
                            const void* pre_save, float* dm, void* dA, void* dB, void* dx, void* ws,
                            size_t ws_bytes, dora_stream_t stream) {
  return backward_impl(false, desc, T, dy, x, W0, A, B, norm, g, su_save, pre_save, dm, dA, dB, dx, ws, ws_bytes,
                       stream);
}

dora_status_t dora_backward_full(const dora_desc_t* desc, int64_t T, const void* dy, const void* x, const void* W0,
                                 const void* A, const void* B, const float* norm, const float* g,
                                 const void* su_save, const void* pre_save, float* dm, void* dA, void* dB, void* dx,
                                 void* ws, size_t ws_bytes, dora_stream_t stream) {
  return backward_impl(true, desc, T, dy, x, W0, A, B, norm, g, su_save, pre_save, dm, dA, dB, dx, ws, ws_bytes,
                       stream);
}

dora_status_t dora_selftest_timeout(uint32_t limit_us, unsigned int* scratch, dora_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) {
    set_error("limit_us must be in 1 .. 1000000");
    return DORA_EINVAL;
  }
  if (!check_ptr(scratch, "scratch", 4)) return DORA_EINVAL;
  return selftest_timeout(limit_us, scratch, reinterpret_cast<cudaStream_t>(stream));
}

dora_status_t dora_device_status(dora_stream_t stream, unsigned int* flags_out) {
  if (!flags_out) {
    set_error("flags_out is NULL");
    return DORA_EINVAL;
  }
  unsigned int v = 0;
  cudaError_t e = read_and_clear_device_status(reinterpret_cast<cudaStream_t>(stream), &v);
  if (e != cudaSuccess) return cuda_status(e, "dora_device_status");
  *flags_out = v;
  if (v) {
    set_error("a kernel's bounded wait ran out");
    return DORA_ETIMEOUT;
  }
  return DORA_OK;
}

const char* dora_last_error(void) { return t_last_error.c_str(); }

int dora_version(void) { return 100; }

}  // extern "C"
