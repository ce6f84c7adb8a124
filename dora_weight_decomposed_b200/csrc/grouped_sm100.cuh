// Grouped persistent GEMM on CTA pairs: one or two GEMMs with the same K
// sources and tile shape in one launch, for GEMMs whose own tiles are too few
// to fill the GPU but which can run side by side (the backward's dB = dz^T su
// and dA^T = x^T du, both K = T). Their output tiles are numbered one after
// the other; pair p of P takes tiles p, p + P, p + 2P, ..., each over its whole
// K, so every tile is stored straight from its accumulator and no partial sum
// leaves the SM. Warp roles as in the persistent pair kernel
// (gemm_sm100.cuh): warp 0 TMA, warp 1 MMA (leader CTA), warps 2-5 epilogue,
// two TMEM accumulators when BN <= 256 so that a tile's epilogue overlaps the
// next tile's MMAs. The output form per problem is a ClusterOut: alpha * acc in
// bf16, row-major or transposed (out[n][m]).
#pragma once

#include "gemm_sm100.cuh"

namespace dora {

struct GroupProblem {
  int M, N;       // output rows and columns
  int n_tiles;    // column tiles (BN wide)
  int tile_base;  // index of the problem's first tile
  ClusterOut o;
};

struct GroupGeom {
  int kb0, kb1;   // k-blocks from source 0 and source 1 (the same for every problem)
  int tiles;      // tiles of all problems
  int nprob;      // 1 or 2
  GroupProblem pr[2];
};

// Tensor maps of up to two problems (source 1 maps repeat source 0 when there is none).
struct GroupMaps {
  CUtensorMap a0[2], a1[2], b0[2], b1[2];
};

template <class Cfg>
struct GroupLayout {
  static constexpr int STAGES_RAW = kSmemBudget / Cfg::STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 3, "stages");
  static constexpr int SMEM_BYTES = STAGES * Cfg::STAGE_BYTES + 256 + 1024;
};

// Problem and tile coordinates of flattened tile t.
__device__ __forceinline__ int group_tile(const GroupGeom& g, int t, int& tm, int& tn) {
  const int j = (g.nprob > 1 && t >= g.pr[1].tile_base) ? 1 : 0;
  const int local = t - g.pr[j].tile_base;
  tm = local / g.pr[j].n_tiles;
  tn = local - tm * g.pr[j].n_tiles;
  return j;
}

template <class Cfg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_sm100_pair_grouped_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupGeom g) {
  constexpr int STAGES = GroupLayout<Cfg>::STAGES;
  constexpr int NACC = Cfg::NUM_ACC;
  constexpr uint32_t ACC_COLS = Cfg::ACC_COLS;
  constexpr uint32_t TMEM_COLS = Cfg::TMEM_COLS;
  constexpr int NCH = Cfg::BN / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;  // [2]
  uint64_t* acce = accf + 2;        // [2], used in the leader only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int KB = g.kb0 + g.kb1;

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 8);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < g.nprob; ++j) {
      prefetch_tmap(&maps.a0[j]);
      prefetch_tmap(&maps.b0[j]);
      if (g.kb1 > 0) {
        prefetch_tmap(&maps.a1[j]);
        prefetch_tmap(&maps.b1[j]);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
#pragma unroll 1
      for (int t = pair; t < g.tiles && ok; t += npairs) {
        int tm, tn;
        const int j = group_tile(g, t, tm, tn);
        const int m0 = tm * 2 * kBM + (int)rank * kBM;
        const int nb0 = tn * Cfg::BN + (int)rank * Cfg::H0;
        const int nb1 = tn * Cfg::BN + Cfg::N0 + (int)rank * Cfg::H1;
#pragma unroll 1
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
          const bool src1 = kb >= g.kb0;
          const int k0 = (src1 ? kb - g.kb0 : kb) * kBK;
          const CUtensorMap* ta = src1 ? &maps.a1[j] : &maps.a0[j];
          const CUtensorMap* tb = src1 ? &maps.b1[j] : &maps.b0[j];
          if (!Cfg::A_MN) {
            tma_load_2d_pair(sa, ta, fb, k0, m0);
          } else {
            tma_load_2d_pair(sa, ta, fb, m0, k0);
            tma_load_2d_pair(sa + 8192, ta, fb, m0 + 64, k0);
          }
#pragma unroll
          for (int q = 0; q < Cfg::B0_LOADS; ++q) {
            if (!Cfg::B_MN)
              tma_load_2d_pair(sb + q * Cfg::B_BOX * 128, tb, fb, k0, nb0 + q * Cfg::B_BOX);
            else
              tma_load_2d_pair(sb + q * 8192, tb, fb, nb0 + q * 64, k0);
          }
#pragma unroll
          for (int q = 0; q < Cfg::B1_LOADS; ++q) {
            if (!Cfg::B_MN)
              tma_load_2d_pair(sb + Cfg::B1_OFFSET + q * Cfg::B_BOX * 128, tb, fb, k0, nb1 + q * Cfg::B_BOX);
            else
              tma_load_2d_pair(sb + Cfg::B1_OFFSET + q * 8192, tb, fb, nb1 + q * 64, k0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc0 = idesc_bf16_f32(2 * kBM, Cfg::N0, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t idesc1 = idesc_bf16_f32(2 * kBM, Cfg::N1 > 0 ? Cfg::N1 : 16, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t a_kstep = Cfg::A_MN ? 2048u : 32u;
      constexpr uint32_t b_kstep = Cfg::B_MN ? 2048u : 32u;
      constexpr uint32_t a_lbo = Cfg::A_MN ? 8192u : 16u;
      constexpr uint32_t b_lbo = Cfg::B_MN ? 8192u : 16u;
      int it = 0, jt = 0;
      bool ok = true;
#pragma unroll 1
      for (int t = pair; t < g.tiles && ok; t += npairs, ++jt) {
        const int b = jt % NACC;
        const uint32_t uph = (uint32_t)(jt / NACC) & 1u;
        if (!mbar_wait(&acce[b], uph ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)b * ACC_COLS;
#pragma unroll 1
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sa + kk * a_kstep, a_lbo, 1024u);
            const uint64_t bd0 = sdesc_sw128(sb + kk * b_kstep, b_lbo, 1024u);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            umma_bf16_pair(d_tmem, ad, bd0, idesc0, acc);
            if (Cfg::N1 > 0) {
              const uint64_t bd1 = sdesc_sw128(sb + Cfg::B1_OFFSET + kk * b_kstep, b_lbo, 1024u);
              umma_bf16_pair(d_tmem + (uint32_t)Cfg::N0, ad, bd1, idesc1, acc);
            }
          }
          umma_commit_pair(&empty[s], 0x3);
        }
        umma_commit_pair(&accf[b], 0x3);
      }
    }
  } else {
    // ---- epilogue: each tile straight from its accumulator, one row per thread
    const int qw = warp & 3;
    const int row = qw * 32 + lane;
    int jt = 0;
#pragma unroll 1
    for (int t = pair; t < g.tiles; t += npairs, ++jt) {
      const int b = jt % NACC;
      const uint32_t uph = (uint32_t)(jt / NACC) & 1u;
      // tcgen05.ld is warp-collective: the whole warp takes the same branch.
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[b], uph))) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t)b * ACC_COLS + ((uint32_t)(qw * 32) << 16);
      int tm, tn;
      const int j = group_tile(g, t, tm, tn);
      const GroupProblem& pr = g.pr[j];
      const ClusterOut& o = pr.o;
      const int m = tm * 2 * kBM + (int)rank * kBM + row;
      const bool row_ok = m < pr.M;
#pragma unroll 1
      for (int c = 0; c < NCH; ++c) {
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), v);
        if (c == NCH - 1) {
          // The whole row is read out of TMEM: hand the accumulator back before storing.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acce[b]), 0));
        }
        if (!row_ok) continue;
        const int n = tn * Cfg::BN + c * 32;
        if (o.transpose) {
          // out[n + i][m]: the warp's 32 consecutive rows m give 64 contiguous bytes per column.
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (n + i < pr.N) o.out[(long long)(n + i) * o.ldo + m] = __float2bfloat16_rn(o.alpha * v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= o.alpha;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (n + 8 * q < pr.N) store_bf16x8(o.out + (long long)m * o.ldo + n + 8 * q, v + 8 * q);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace dora
