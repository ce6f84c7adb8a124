// Merged weight W' = diag(g) (W0 + s B A) on CTA pairs (DoRA notes,
// Algorithm 1 steps 16-17: fold magnitude and low-rank update into one dense
// weight for deployment).
//
// The product B A has K = r only, so per output element the kernel moves four
// bytes of HBM (W0 in, W' out) for 2r flops: HBM traffic, tensor-core time and
// the operand traffic from L2 are all of the same size and have to overlap.
//
// A cluster of two CTAs computes 256 x 256 tiles of B A with tcgen05.mma
// cta_group::2 into one of two TMEM accumulators; the TMA engine only moves
// the operands (L2-resident). Pairs take tiles round-robin in row-major
// order, so the tiles in flight at any moment sit side by side in a few row
// bands: their W0 rows are read and written nearly whole at the same time,
// which keeps the DRAM pages they open busy.
//
// W0 is streamed by the epilogue warps themselves: each copies its own
// 32 x 32 pieces of W0 with cp.async into a private ring DEPTH chunks ahead,
// four lanes per 64-byte row piece. (A TMA slab ring fed by a producer warp
// measured no faster and needs a warp and two barriers per slab more.) The thread that owns a TMEM row then combines
// its row (w <- g (w + s acc), rounded to bf16 once) in place and the warp
// writes the piece back row-contiguously with plain coalesced stores; no
// proxy fence and no completion wait sits on that path. The epilogue is
// latency-bound per warp, so two warps share each TMEM lane quarter, each
// taking one 32-column half of every 64-column chunk.
//
// Warps: 0 operand TMA, 1 MMA (leader CTA), 2-9 epilogue.
#pragma once

#include "gemm_sm100.cuh"

namespace dora {

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// STAGES: operand stages (128 rows of B and 128 columns of A per k-block);
// DEPTH: W0 chunks each epilogue warp keeps in flight.
template <int STAGES_, int DEPTH_>
struct MergeCfg {
  static constexpr int STAGES = STAGES_;
  static constexpr int DEPTH = DEPTH_;
  static constexpr int BN = 256;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
  static constexpr int A_STAGE_BYTES = kBM * kBK * 2;       // 128 rows of B x 64 k of bf16: 16 KB
  static constexpr int B_STAGE_BYTES = (BN / 2) * kBK * 2;  // this CTA's 128 columns of A x 64 k: 16 KB
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int CHUNKS = BN / 64;                    // 64-column chunks per tile
  static constexpr int PIECE_BYTES = 32 * 64;               // one warp's 32 rows x 32 bf16
  static constexpr int RING_BYTES = EPI_WARPS * DEPTH * PIECE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + RING_BYTES + BAR_BYTES + 1024;
  static_assert(SMEM_BYTES <= 232448, "merge kernel shared memory");
  static_assert(STAGES >= 2 && DEPTH >= 2, "merge rings");
  static constexpr uint32_t ACC_COLS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
};

// The configuration dora_merge launches: 4 operand stages (128 KB), a ring of
// 6 W0 pieces per epilogue warp (96 KB); one CTA pair per two SMs, at most
// one per tile.
using MergeLaunchCfg = MergeCfg<4, 6>;
inline long long merge_pairs(long long tiles, int sms) {
  return tiles < sms / 2 ? (tiles > 0 ? tiles : 1) : (sms / 2 > 0 ? sms / 2 : 1);
}

struct MergeGeom {
  int M, N, kb;  // d_out, d_in, k-blocks of r
  const float* g;
  float s;
  const __nv_bfloat16* W0;  // [M x N], row stride N
  __nv_bfloat16* out;       // W' [M x N], row stride N; may be W0
};

// Offset of 16-byte unit k of row lr inside a 32 x 64-byte piece (units
// swizzled by bits 1-2 of the row, so that both a row per lane and four lanes
// per row touch every bank group once per 512 bytes).
__device__ __forceinline__ uint32_t piece_off(int lr, int k) {
  return (uint32_t)(lr * 64) + ((((uint32_t)k) ^ (((uint32_t)lr >> 1) & 3u)) << 4);
}

template <class Cfg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg::THREADS, 1)
    merge_pair_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                      const MergeGeom geom) {
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;                               // rows of B, columns of A
  uint8_t* rings = stages + STAGES * Cfg::STAGE_BYTES;  // W0 pieces, DEPTH per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(rings + Cfg::RING_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;  // [2]
  uint64_t* acce = accf + 2;        // [2], leader only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int m_tiles = (geom.M + 2 * kBM - 1) / (2 * kBM);
  const int n_tiles = (geom.N + Cfg::BN - 1) / Cfg::BN;
  // Tiles of this pair: first, first + step, ... below last (row-major tile list).
  const int first = blockIdx.x >> 1;
  const int last = m_tiles * n_tiles;
  const int step = gridDim.x >> 1;

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 2 * Cfg::EPI_WARPS);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tA);
    prefetch_tmap(&tB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
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
    // Per k-block: this CTA's 128 rows of B and its 128 columns of A.
    if (lane == 0) {
      int it = 0;
      bool ok = true;
#pragma unroll 1
      for (int item = first; item < last && ok; item += step) {
        const int tm = item / n_tiles, tn = item - tm * n_tiles;
        const int m0 = tm * 2 * kBM + (int)rank * kBM;
        const int nb = tn * Cfg::BN + (int)rank * (Cfg::BN / 2);
#pragma unroll 1
        for (int kb = 0; kb < geom.kb; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((uint32_t)(it / STAGES) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          uint8_t* sb = stages + s * Cfg::STAGE_BYTES;
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * Cfg::STAGE_BYTES);
          tma_load_2d_pair(sb, &tA, fb, kb * kBK, m0);
          sb += Cfg::A_STAGE_BYTES;
#pragma unroll
          for (int j = 0; j < Cfg::BN / 128; ++j) tma_load_2d_pair(sb + j * 8192, &tB, fb, nb + j * 64, kb * kBK);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, Cfg::BN, false, true);
      int it = 0, j = 0;
      bool ok = true;
#pragma unroll 1
      for (int item = first; item < last && ok; item += step, ++j) {
        const int b = j & 1;
        if (!mbar_wait(&acce[b], ((uint32_t)(j >> 1) & 1u) ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)b * Cfg::ACC_COLS;
#pragma unroll 1
        for (int kb = 0; kb < geom.kb; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (uint32_t)(it / STAGES) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + (uint32_t)Cfg::A_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sa + kk * 32u, 16u, 1024u);
            const uint64_t bd = sdesc_sw128(sb + kk * 2048u, 8192u, 1024u);
            umma_bf16_pair(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty[s], 0x3);
        }
        umma_commit_pair(&accf[b], 0x3);
      }
    }
  } else {
    // Epilogue warp: TMEM lane quarter q (rows 32 q .. 32 q + 31), column half h of each chunk.
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    uint8_t* ring = rings + (warp - 2) * Cfg::DEPTH * Cfg::PIECE_BYTES;
    // Copy lanes: four per row piece, rows (lane >> 2) + 8 i, 16-byte unit (lane & 3).
    const int ck = lane & 3;
    // W0 piece prefetch: (item, chunk) of the next piece to fetch, and its ring slot.
    int f_item = first, f_c = 0, f_n = 0;
    auto fetch = [&]() {
      if (f_item < last) {
        const int tm = f_item / n_tiles, tn = f_item - tm * n_tiles;
        const int r0 = tm * 2 * kBM + (int)rank * kBM + q * 32 + (lane >> 2);
        const int col = tn * Cfg::BN + 64 * f_c + 32 * h + 8 * ck;
        uint8_t* piece = ring + (f_n % Cfg::DEPTH) * Cfg::PIECE_BYTES;
        const __nv_bfloat16* src = geom.W0 + (long long)r0 * geom.N + col;
        const bool col_in = col < geom.N;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool in = col_in && r0 + 8 * i < geom.M;
          cp_async16(piece + piece_off((lane >> 2) + 8 * i, ck), in ? src + (long long)(8 * i) * geom.N : geom.W0,
                     in ? 16u : 0u);
        }
        if (++f_c == Cfg::CHUNKS || tn * Cfg::BN + 64 * f_c >= geom.N) {
          f_c = 0;
          f_item += step;
        }
        ++f_n;
      }
      cp_async_commit();  // one group per call, empty past the end, so group counts stay aligned
    };
#pragma unroll 1
    for (int d = 0; d < Cfg::DEPTH - 1; ++d) fetch();

    int n = 0, j = 0;
    bool ok = true;
#pragma unroll 1
    for (int item = first; item < last && ok; item += step, ++j) {
      const int b = j & 1;
      const int tm = item / n_tiles, tn = item - tm * n_tiles;
      const int m0 = tm * 2 * kBM + (int)rank * kBM;
      const int n0 = tn * Cfg::BN;
      const int m = m0 + q * 32 + lane;
      const float gm = m < geom.M ? geom.g[m] : 0.f;
      if (!mbar_wait(&accf[b], (uint32_t)(j >> 1) & 1u)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t)b * Cfg::ACC_COLS + ((uint32_t)(q * 32) << 16) + (uint32_t)(32 * h);
#pragma unroll 1
      for (int c = 0; c < Cfg::CHUNKS && n0 + 64 * c < geom.N; ++c, ++n) {
        fetch();  // piece n + DEPTH - 1
        float v[32];
        tmem_ld32(taddr + (uint32_t)(64 * c), v);
        cp_async_wait<Cfg::DEPTH - 1>();  // piece n has landed (this lane's copies)
        __syncwarp();                     // ... and every other lane's
        uint8_t* piece = ring + (n % Cfg::DEPTH) * Cfg::PIECE_BYTES;
        // All loads first, then the math, then all stores: the four units are
        // independent and their latencies overlap.
        uint4 raw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) raw[k] = *reinterpret_cast<const uint4*>(piece + piece_off(lane, k));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&raw[k]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 w = __bfloat1622float2(hv[i]);
            hv[i] = __floats2bfloat162_rn(gm * fmaf(geom.s, v[8 * k + 2 * i], w.x),
                                          gm * fmaf(geom.s, v[8 * k + 2 * i + 1], w.y));
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(piece + piece_off(lane, k)) = raw[k];
        __syncwarp();
        const int col = n0 + 64 * c + 32 * h + 8 * ck;
        const int gr0 = m0 + q * 32 + (lane >> 2);
        uint4 val[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) val[i] = *reinterpret_cast<const uint4*>(piece + piece_off((lane >> 2) + 8 * i, ck));
        __nv_bfloat16* dst = geom.out + (long long)gr0 * geom.N + col;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (gr0 + 8 * i < geom.M && col < geom.N) *reinterpret_cast<uint4*>(dst + (long long)(8 * i) * geom.N) = val[i];
        __syncwarp();  // the piece is refilled DEPTH - 1 chunks later
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acce[b]), 0));
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace dora
