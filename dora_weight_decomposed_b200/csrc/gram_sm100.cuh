// Gram matrix of the factored norm, G = A A^T, in one launch on sm_100a.
//
// The norm's Gram term s^2 B_i G B_i^T enters the norm GEMM as a K-extension
// [B | B] [Gs_hi | Gs_lo]^T with Gs = scale * G split into bf16 hi + lo parts
// (Scaling DoRA abstract: the Gram term of the factored row norm). This kernel
// writes Gs directly: no fp32 partials in global memory and no second pass.
//
//   * G is symmetric: only the 128 x 128 tiles (ti, tj) with ti <= tj are
//     computed; the epilogue writes tile (tj, ti) transposed. A diagonal tile
//     loads each A k-block once and uses it as both MMA operands.
//   * Each tile is one cluster of CS CTAs (cluster rank = K slice). Every CTA
//     runs tcgen05 MMAs over its slice into TMEM, drains the accumulator into
//     its own shared memory, and after a cluster barrier reduces 128 / CS rows
//     of the tile by reading the same rows of every CTA of the cluster through
//     distributed shared memory, always in rank order (the result does not
//     depend on timing). CS is chosen per call: few CTAs when the norm GEMM
//     that follows leaves SMs free for them (the Gram then runs beside its W0
//     main loop), else eight for the shortest Gram.
//   * Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
//     issues the MMAs, warps 2-5 drain TMEM; all six warps reduce.
//   * Dependent launch: the kernel waits for its predecessor before it
//     triggers its dependent, so the norm GEMM that follows may start its W0
//     main loop at once and only waits for this grid before loading Gs.
//     Before triggering, block (0, 0) zeroes the norm GEMM's split counters.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

constexpr int kGramTile = 128;
constexpr int kGramStages = 6;
constexpr int kGramOpBytes = kGramTile * 64 * 2;      // one 128-row x 64-column bf16 k-block (16 KB)
constexpr int kGramStageBytes = 2 * kGramOpBytes;
constexpr int kGramRedLd = kGramTile + 4;             // fp32 row stride of the reduction buffer (floats)
constexpr int kGramSmemBytes = kGramStages * kGramStageBytes + 256 + 1024;
constexpr int kGramTrOffset = 128 * 1024;             // transposed bf16 staging (after the fp32 buffer)
static_assert(kGramTile * kGramRedLd * 4 <= kGramStages * kGramStageBytes, "reduction buffer fits the ring");

struct GramParams {
  int r;              // rank (rows of A)
  int rp;             // r rounded up to 64: column count of each half of gs2
  int nt;             // 128-row blocks of A
  int kb_total;       // k-blocks of 64 columns over d_in
  int kps;            // k-blocks per cluster rank
  float scale;        // Gs = scale * G
  __nv_bfloat16* gs2; // [r x 2 rp]: [hi | lo], zero in columns r .. rp - 1 of each half
  unsigned int* zero_words;  // words the next kernel needs zeroed (may be null)
  int zero_count;
};

// Tile t of the upper triangle (ti <= tj), row-major over ti.
__device__ __forceinline__ void gram_tile(int t, int nt, int& ti, int& tj) {
  ti = 0;
  int first = 0;
  while (t >= first + (nt - ti)) {
    first += nt - ti;
    ++ti;
  }
  tj = ti + (t - first);
}

template <int CS>
__global__ void __launch_bounds__(192, 1) gram_cluster_kernel(const __grid_constant__ CUtensorMap tA,
                                                              const GramParams p) {
  static_assert(kGramTile % CS == 0 && CS <= 8, "rows split evenly over the cluster");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGramStages * kGramStageBytes);
  uint64_t* empty = full + kGramStages;
  uint64_t* accf = empty + kGramStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  float* red = reinterpret_cast<float*>(smem);  // after the main loop: [128][kGramRedLd] fp32

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  int ti, tj;
  gram_tile(blockIdx.y, p.nt, ti, tj);
  const bool diag = ti == tj;
  const int kb_begin = (int)crank * p.kps;
  const int kb_end = min(p.kb_total, kb_begin + p.kps);
  const int nkb = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tA);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The predecessor has completed (A is final, the counters' last users are done)
  // before anything is read, zeroed or triggered.
  pdl_wait();
  if (blockIdx.x == 0 && blockIdx.y == 0 && p.zero_words) {
    for (int i = threadIdx.x; i < p.zero_count; i += blockDim.x) p.zero_words[i] = 0u;
    __threadfence();
  }
  pdl_trigger();

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = diag ? (uint32_t)kGramOpBytes : (uint32_t)kGramStageBytes;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kGramStages;
        if (!mbar_wait(&empty[s], ((uint32_t)(i / kGramStages) & 1u) ^ 1u)) break;
        uint8_t* sa = smem + s * kGramStageBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        const int k0 = (kb_begin + i) * 64;
        tma_load_2d(sa, &tA, &full[s], k0, ti * kGramTile);
        if (!diag) tma_load_2d(sa + kGramOpBytes, &tA, &full[s], k0, tj * kGramTile);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGramTile, kGramTile, false, false);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kGramStages;
        if (!mbar_wait(&full[s], (uint32_t)(i / kGramStages) & 1u)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * kGramStageBytes);
        const uint32_t sb = diag ? sa : sa + (uint32_t)kGramOpBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
    }
    __syncwarp();
  } else {
    // Drain this warp's 32 accumulator rows into the reduction buffer (zeros if the slice was empty).
    const int row = (warp & 3) * 32 + lane;
    // tcgen05.ld is warp-collective: the whole warp takes the same branch below.
    ok = __all_sync(0xffffffffu, mbar_wait(accf, 0));
    tc_fence_after();
    float* dst = red + row * kGramRedLd;
#pragma unroll 1
    for (int col = 0; col < kGramTile; col += 32) {
      float v[32];
      if (nkb > 0 && ok) {
        tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)col, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + col + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
  }
  tc_fence_before();
  cluster_sync();  // every CTA's buffer is complete and visible to the cluster

  // Rows [crank * kRows, +kRows) of the tile: the cluster's slices summed in rank order,
  // read through generic pointers so that all CS loads of an item are in flight at once.
  constexpr int kRows = kGramTile / CS;
  const float* srcs[CS];
#pragma unroll
  for (int z = 0; z < CS; ++z) srcs[z] = z == (int)crank ? red : dsmem_ptr(red, (uint32_t)z);  // own: local
  const int two_rp = 2 * p.rp;
  // Staging of the transposed tile (after the fp32 buffer in the idle ring).
  constexpr int kTrLd = kRows + 8;  // bf16 row stride, 16-byte aligned
  __nv_bfloat16* tr_hi = reinterpret_cast<__nv_bfloat16*>(smem + kGramTrOffset);
  __nv_bfloat16* tr_lo = tr_hi + kGramTile * kTrLd;
  static_assert(kGramTile * kGramRedLd * 4 <= kGramTrOffset &&
                    kGramTrOffset + 2 * kGramTile * kTrLd * 2 <= kGramStages * kGramStageBytes,
                "transposed staging fits the ring after the fp32 buffer");
  // Four items per thread per batch: all their remote loads are issued before any is summed.
  // A single tile (r <= 128, diagonal, nothing to transpose) spreads only its r valid rows and
  // rp columns over the cluster, so small ranks do not reduce the zero padding of the tile.
  const bool single = p.nt == 1;
  const int rows_per = single ? (p.r + CS - 1) / CS : kRows;
  const int row_lo = (int)crank * rows_per;
  const int rows_here = single ? max(0, min(p.r, row_lo + rows_per) - row_lo) : kRows;
  const int cols4 = single ? p.rp / 4 : kGramTile / 4;  // 4-column items per row
  const int n_items = rows_here * cols4;
  constexpr int kU = 4;
  for (int idx0 = threadIdx.x; idx0 < n_items; idx0 += 192 * kU) {
    float4 vv[kU][CS];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int idx = idx0 + u * 192;
      if (idx < n_items) {
        const int off = (row_lo + idx / cols4) * kGramRedLd + (idx % cols4) * 4;
#pragma unroll
        for (int z = 0; z < CS; ++z) vv[u][z] = *reinterpret_cast<const float4*>(srcs[z] + off);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int idx = idx0 + u * 192;
      if (idx >= n_items) break;
      const int lr = row_lo + idx / cols4;
      const int lc = (idx % cols4) * 4;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int z = 0; z < CS; ++z) {
        a.x += vv[u][z].x;
        a.y += vv[u][z].y;
        a.z += vv[u][z].z;
        a.w += vv[u][z].w;
      }
      const float xs[4] = {p.scale * a.x, p.scale * a.y, p.scale * a.z, p.scale * a.w};
      const int gi = ti * kGramTile + lr;
      const int gj = tj * kGramTile + lc;
      __nv_bfloat16 hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool valid = gi < p.r && gj + j < p.r;  // outside r: zero (the padding of gs2)
        const __nv_bfloat16 h = __float2bfloat16_rn(valid ? xs[j] : 0.f);
        hi[j] = h;
        lo[j] = __float2bfloat16_rn(valid ? xs[j] - __bfloat162float(h) : 0.f);
      }
      if (!diag) {
        // The transposed values, staged so that tile (tj, ti) is written in whole rows below.
        const int lrl = lr - row_lo;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tr_hi[(lc + j) * kTrLd + lrl] = hi[j];
          tr_lo[(lc + j) * kTrLd + lrl] = lo[j];
        }
      }
      if (gi >= p.r) continue;  // (the next item of the batch)
      __nv_bfloat16* rowp = p.gs2 + (size_t)gi * two_rp;
      if (gj + 3 < p.rp) {
        *reinterpret_cast<uint2*>(rowp + gj) = *reinterpret_cast<const uint2*>(hi);
        *reinterpret_cast<uint2*>(rowp + p.rp + gj) = *reinterpret_cast<const uint2*>(lo);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (gj + j < p.rp) {
            rowp[gj + j] = hi[j];
            rowp[p.rp + gj + j] = lo[j];
          }
      }
    }
  }
  if (!diag) {
    // G is symmetric: rows tj * 128 + c of gs2 receive this CTA's kRows columns
    // ti * 128 + crank * kRows .. as contiguous 16-byte pieces (hi, then lo).
    __syncthreads();
    const int gi0 = ti * kGramTile + (int)crank * kRows;
    constexpr int kPieces = kRows / 8;
    for (int idx = threadIdx.x; idx < kGramTile * kPieces * 2; idx += blockDim.x) {
      const int half = idx / (kGramTile * kPieces);
      const int rem = idx - half * kGramTile * kPieces;
      const int c = rem / kPieces;
      const int pc = (rem - c * kPieces) * 8;
      const int R = tj * kGramTile + c;
      if (R >= p.r || gi0 + pc >= p.rp) continue;
      const __nv_bfloat16* src = (half ? tr_lo : tr_hi) + c * kTrLd + pc;
      *reinterpret_cast<uint4*>(p.gs2 + (size_t)R * two_rp + (half ? p.rp : 0) + gi0 + pc) =
          *reinterpret_cast<const uint4*>(src);
    }
  }
  cluster_sync();  // no CTA leaves while another still reads its buffer
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  (void)ok;
}

}  // namespace dora
