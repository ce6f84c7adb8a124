// Warp-specialised tcgen05 GEMM core for sm_100a.
//
//   D[M x N] = sum over k of Aop[m, k] * Bop[n, k]      (fp32 accumulator in TMEM)
//
// Aop is 128 rows per CTA, Bop is BN rows per CTA, K is streamed in blocks of
// 64 bf16 (one 128-byte swizzle row) through a STAGES-deep shared-memory ring
// filled by TMA. Either operand may be stored K-major (rows of K contiguous) or
// MN-major (rows of M/N contiguous, e.g. a token-major tensor used with K = T).
// K may come from two sources back to back (source 0 then source 1, e.g.
// [x | s*u] against [W0 | B]); each source has its own tensor maps. Source 1
// of A may be re-read cyclically (a1_kwrap) to pair one A block with several
// B blocks, e.g. [B | B] against [G_hi | G_lo].
// blockIdx = (n tile, m tile, K split).
//
// Warp roles (192 threads):
//   warp 0     one lane issues the TMA loads for each stage
//   warp 1     allocates TMEM; one lane issues tcgen05.mma and commits
//   warps 2-5  epilogue: warp w owns TMEM lanes 32*(w%4) .. +31 (= tile rows);
//              an epilogue may also read each A stage (kReadsA) before it is
//              released (the CTA-pair split kernel below does the same for the
//              norm's row sums of squares).
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 192;
constexpr int kSmemBudget = 200 * 1024;

struct GemmGeom {
  int M;             // valid output rows
  int N;             // valid output columns
  int kb0;           // k-blocks taken from source 0
  int kb1;           // k-blocks taken from source 1
  int kb_per_split;  // k-blocks per blockIdx.z
  int a1_kwrap;      // > 0: source-1 A coordinates wrap modulo this many K elements
  // CTA-pair kernels (persistent, split, cluster): nonzero when only the source-1
  // operands come from the preceding grid. The kernel then starts its source-0
  // main loop at once; the producer waits for the preceding grid just before its
  // first source-1 load, and the epilogue (or the cluster reduction) before it
  // writes anything. Only valid after a grid that waits for its own predecessor
  // before it triggers (wait_then_trigger, or the Gram kernel), so that all work
  // before that grid is complete when this one starts.
  int defer_wait_src1 = 0;
  // Persistent and cluster kernels: wait for the preceding grid before letting
  // the dependent grid launch (see defer_wait_src1).
  int wait_then_trigger = 0;
};

// The dependent-launch handshake at the end of a CTA-pair kernel's prologue.
__device__ __forceinline__ void pdl_handshake(const GemmGeom& geom) {
  if (geom.wait_then_trigger) {
    pdl_wait();
    pdl_trigger();
  } else {
    pdl_trigger();
    if (!geom.defer_wait_src1) pdl_wait();
  }
}

template <int BN_, bool A_MN_, bool B_MN_>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 512, "BN");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-wide swizzle chunks");
  static_assert(BN <= 128 || BN % 64 == 0, "BN above 128 must be a multiple of 64");
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "stages");
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : BN <= 256 ? 256 : 512;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr int MMA_N0 = BN <= 256 ? BN : 256;
  static constexpr int MMA_N1 = BN <= 256 ? 0 : BN - 256;
  // TMA boxes: K-major B uses boxes of B_BOX rows; MN-major uses 64x64 chunks.
  static constexpr int B_BOX = B_MN ? 64 : (BN <= 128 ? BN : (BN % 128 == 0 ? 128 : 64));
  static constexpr int B_LOADS = BN / B_BOX;
};

struct EpiCtx {
  uint32_t taddr;  // TMEM address of this warp's lane quarter, column 0
  int row;         // row within the tile (0..127) owned by this thread
  int m;           // global output row
  int n0;          // first global output column of the tile
  int split;       // blockIdx.z
  bool has_acc;    // false when this split had no k-blocks (accumulator never written)
  // Non-persistent kernels only (one CTA per tile, or the CTA-pair split
  // kernel): once the accumulator is complete the stage ring is idle, and an
  // epilogue may refill it through its own barrier.
  uint8_t* stage_smem;        // start of the stage ring
  int stage_bytes;            // bytes of the ring
  uint64_t* aux_bar;          // spare mbarrier (count 1), phase 0 unused so far
  const CUtensorMap* tA1;     // A-operand source-1 tensor map
  // CTA-pair split kernel with an epilogue that has its A source-1 rows
  // prefetched (Epi::kRefillA1): 16 KB slab sl sits in ring stage
  // (refill_first + sl / (stage_stride / 16384)) % ring_stages, at
  // (sl % (stage_stride / 16384)) * 16384 bytes, complete on aux_bar phase 0.
  int refill_first;
  int ring_stages;
  int stage_stride;
  // K-split bookkeeping (non-persistent kernels): the output rows' index (one
  // per 128-row block), the number of splits, and a shared-memory word for
  // the last-split decision.
  int tile_id;
  int splits;
  uint32_t* flag;
};

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, const float* v) {
  __nv_bfloat162 p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(p);
}

// The same with the streaming (evict-first) cache hint: for outputs no kernel
// of the call reads again, so that their lines leave L2 early and make room
// for the data the next kernel reads.
__device__ __forceinline__ void store_bf16x8_cs(__nv_bfloat16* dst, const float* v) {
  __nv_bfloat162 p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
               : "memory");
}

// Four consecutive bf16 (8 bytes), plain and streaming.
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, float a, float b, float c, float d) {
  __nv_bfloat162 p[2] = {__floats2bfloat162_rn(a, b), __floats2bfloat162_rn(c, d)};
  *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(p);
}
__device__ __forceinline__ void store_bf16x4_cs(__nv_bfloat16* dst, float a, float b, float c, float d) {
  __nv_bfloat162 p[2] = {__floats2bfloat162_rn(a, b), __floats2bfloat162_rn(c, d)};
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  asm volatile("st.global.cs.v2.b32 [%0], {%1, %2};" ::"l"(dst), "r"(w.x), "r"(w.y) : "memory");
}

// 16-column TMEM load (for tiles whose width is an odd multiple of 16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Visit the thread's accumulator row in chunks of 32 columns: f(col, v[32]).
// A trailing 16-wide chunk is zero-padded to 32. Warp-collective.
template <int BN, class F>
__device__ __forceinline__ void for_each_acc_chunk(const EpiCtx& c, F&& f) {
#pragma unroll 1
  for (int col = 0; col < BN; col += 32) {
    float v[32];
    if (BN - col >= 32) {
      if (c.has_acc) {
        tmem_ld32(c.taddr + col, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
    } else {
      if (c.has_acc) {
        tmem_ld16(c.taddr + col, v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 16; i < 32; ++i) v[i] = 0.f;
    }
    f(col, v);
  }
}

template <class Cfg, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                      const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
                      const GemmGeom geom, const typename Epi::Params ep) {
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* aux = accf + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int m_tile = blockIdx.y;
  const int split = blockIdx.z;
  const int kb_total = geom.kb0 + geom.kb1;
  const int kb_begin = split * geom.kb_per_split;
  const int kb_end = min(kb_total, kb_begin + geom.kb_per_split);
  const int nkb = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + (Epi::kReadsA ? 4 : 0));
    }
    mbar_init(accf, 1);
    mbar_init(aux, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tA0);
    prefetch_tmap(&tB0);
    if (geom.kb1 > 0) {
      prefetch_tmap(&tA1);
      prefetch_tmap(&tB1);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u)) break;
        uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
        uint8_t* sb = sa + Cfg::A_BYTES;
        mbar_arrive_expect_tx(&full[s], Cfg::STAGE_BYTES);
        const int kb = kb_begin + i;
        const bool src1 = kb >= geom.kb0;
        const int k0 = (src1 ? kb - geom.kb0 : kb) * kBK;
        const int k0a = (src1 && geom.a1_kwrap > 0) ? k0 % geom.a1_kwrap : k0;
        const CUtensorMap* ta = src1 ? &tA1 : &tA0;
        const CUtensorMap* tb = src1 ? &tB1 : &tB0;
        const int m0 = m_tile * kBM;
        const int n0 = n_tile * Cfg::BN;
        if (!Cfg::A_MN) {
          tma_load_2d(sa, ta, &full[s], k0a, m0);
        } else {
          tma_load_2d(sa, ta, &full[s], m0, k0a);
          tma_load_2d(sa + 8192, ta, &full[s], m0 + 64, k0a);
        }
#pragma unroll
        for (int j = 0; j < Cfg::B_LOADS; ++j) {
          if (!Cfg::B_MN)
            tma_load_2d(sb + j * Cfg::B_BOX * 128, tb, &full[s], k0, n0 + j * Cfg::B_BOX);
          else
            tma_load_2d(sb + j * 8192, tb, &full[s], n0 + j * 64, k0);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc0 = idesc_bf16_f32(kBM, Cfg::MMA_N0, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t idesc1 = idesc_bf16_f32(kBM, Cfg::MMA_N1 > 0 ? Cfg::MMA_N1 : 16, Cfg::A_MN, Cfg::B_MN);
      // Per 16-wide K step: K-major advances 32 bytes inside the swizzle row,
      // MN-major advances 16 rows of 128 bytes.
      constexpr uint32_t a_kstep = Cfg::A_MN ? 2048u : 32u;
      constexpr uint32_t b_kstep = Cfg::B_MN ? 2048u : 32u;
      constexpr uint32_t a_lbo = Cfg::A_MN ? 8192u : 16u;
      constexpr uint32_t b_lbo = Cfg::B_MN ? 8192u : 16u;
      // Offset of the second MMA's B rows (columns 256..): 256 K-major rows or 4 MN-major chunks.
      constexpr uint32_t b_half = Cfg::B_MN ? 4u * 8192u : 256u * 128u;
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sa + kk * a_kstep, a_lbo, 1024u);
          const uint64_t bd0 = sdesc_sw128(sb + kk * b_kstep, b_lbo, 1024u);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_bf16(tmem, ad, bd0, idesc0, acc);
          if (Cfg::MMA_N1 > 0) {
            const uint64_t bd1 = sdesc_sw128(sb + b_half + kk * b_kstep, b_lbo, 1024u);
            umma_bf16(tmem + 256u, ad, bd1, idesc1, acc);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    typename Epi::RowState st{};
    if (Epi::kReadsA) {
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph)) break;
        const int kb = kb_begin + i;
        Epi::on_a_stage(ep, st, smem + s * Cfg::STAGE_BYTES + row * 128, kb >= geom.kb0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    mbar_wait(accf, 0);
    tc_fence_after();
    EpiCtx c;
    c.taddr = tmem + ((uint32_t)(q * 32) << 16);
    c.row = row;
    c.m = m_tile * kBM + row;
    c.n0 = n_tile * Cfg::BN;
    c.split = split;
    c.has_acc = nkb > 0;
    c.stage_smem = smem;
    c.stage_bytes = STAGES * Cfg::STAGE_BYTES;
    c.aux_bar = aux;
    c.tA1 = &tA1;
    c.refill_first = nkb;
    c.ring_stages = STAGES;
    c.stage_stride = Cfg::STAGE_BYTES;
    c.tile_id = m_tile * (int)gridDim.x + n_tile;
    c.splits = (int)gridDim.z;
    c.flag = tmem_slot + 1;
    Epi::template run<Cfg::BN>(ep, st, c, geom);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ tile order
//
// Persistent kernels walk the output tiles t = first, first + step, ... in
// groups of kGroupM m-tiles (m fastest inside a group), so the tiles in flight
// at one time share their A rows and B columns in L2.
constexpr int kGroupM = 8;

__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int& m, int& n) {
  const int per_group = kGroupM * n_tiles;
  const int grp = t / per_group;
  const int first_m = grp * kGroupM;
  const int gm = min(kGroupM, m_tiles - first_m);
  const int rem = t - grp * per_group;
  m = first_m + rem % gm;
  n = rem / gm;
}

// ------------------------------------------------------------------ CTA-pair persistent variant
//
// A cluster of two CTAs computes 256 x BN output tiles with tcgen05.mma
// cta_group::2: each CTA stages its own 128 rows of A and half of the B tile
// (BN/2 rows), so per-SM operand traffic and shared memory per stage drop and
// the ring gets deeper. Both CTAs' TMA loads complete on the leader CTA's
// full barrier; the leader issues the MMAs and commits to the empty and
// accumulator barriers of both CTAs; each CTA's epilogue drains its own TMEM
// rows and reports to the leader. Tiles are walked persistently as above.
template <int BN_, bool A_MN_, bool B_MN_>
struct PairCfg {
  static constexpr int BN = BN_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 512, "pair tile N");
  // N above 256 takes two MMAs: columns [0, N0) and [N0, BN). Each CTA stages
  // half of each MMA's B columns: H0 rows for the first, then H1 for the second.
  static constexpr int N0 = BN <= 256 ? BN : 256;
  static constexpr int N1 = BN - N0;
  static constexpr int H0 = N0 / 2;
  static constexpr int H1 = N1 / 2;
  static constexpr int BH = H0 + H1;
  static_assert(!B_MN || (H0 % 64 == 0 && H1 % 64 == 0), "MN-major B halves are whole 64-wide chunks");
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BH * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr int B_BOX = B_MN ? 64 : (H1 == 0 ? H0 : (H0 == H1 ? H0 : 64));
  static constexpr int B0_LOADS = H0 / B_BOX;
  static constexpr int B1_LOADS = H1 / B_BOX;
  // Offset of the second MMA's B half inside the stage.
  static constexpr uint32_t B1_OFFSET = B_MN ? (uint32_t)(H0 / 64) * 8192u : (uint32_t)H0 * 128u;
  // Two accumulators (epilogue overlaps the next item's MMAs) when N <= 256.
  static constexpr int NUM_ACC = BN <= 256 ? 2 : 1;
  static constexpr uint32_t ACC_COLS = BN <= 64 ? 64 : BN <= 128 ? 128 : BN <= 256 ? 256 : 512;
  static constexpr uint32_t TMEM_COLS = NUM_ACC * ACC_COLS > 512 ? 512 : NUM_ACC * ACC_COLS;
};

// Work items are (output tile, K split) pairs: item = tile * splits + split.
// Shared memory of a pair kernel: the stage ring, the epilogue's own staging
// area (Epi::kStageOutBytes, if any), then the barriers.
template <class Cfg, class Epi>
struct PairLayout {
  static constexpr int EPI_BYTES = Epi::kStageOutBytes;
  static constexpr int STAGES_RAW = (kSmemBudget - EPI_BYTES) / Cfg::STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "stages");
  static constexpr int SMEM_BYTES = STAGES * Cfg::STAGE_BYTES + EPI_BYTES + Cfg::BAR_BYTES + 1024;
};

template <class Cfg, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_sm100_pair_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                           const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
                           const GemmGeom geom, const __grid_constant__ typename Epi::Params ep) {
  static_assert(!Epi::kReadsA, "pair epilogues do not read A stages");
  constexpr int STAGES = PairLayout<Cfg, Epi>::STAGES;
  constexpr int EPI_BYTES = PairLayout<Cfg, Epi>::EPI_BYTES;
  constexpr int NACC = Cfg::NUM_ACC;
  constexpr uint32_t ACC_COLS = Cfg::ACC_COLS;
  constexpr uint32_t TMEM_COLS = Cfg::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;  // [2]
  uint64_t* acce = accf + 2;        // [2], used in the leader only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int m_tiles = (geom.M + 2 * kBM - 1) / (2 * kBM);
  const int n_tiles = (geom.N + Cfg::BN - 1) / Cfg::BN;
  const int kb_total = geom.kb0 + geom.kb1;
  const int kps = geom.kb_per_split;
  const int splits = (kb_total + kps - 1) / kps;
  const int items = m_tiles * n_tiles * splits;

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
    prefetch_tmap(&tA0);
    prefetch_tmap(&tB0);
    if (geom.kb1 > 0) {
      prefetch_tmap(&tA1);
      prefetch_tmap(&tB1);
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
  pdl_handshake(geom);
  const bool defer = geom.defer_wait_src1 != 0 && !geom.wait_then_trigger;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      bool waited = !defer;
#pragma unroll 1
      for (int item = pair; item < items && ok; item += npairs) {
        const int t = item / splits, split = item - t * splits;
        int tm, tn;
        tile_coords(t, m_tiles, n_tiles, tm, tn);
        const int m0 = tm * 2 * kBM + (int)rank * kBM;
        const int nb0 = tn * Cfg::BN + (int)rank * Cfg::H0;
        const int nb1 = tn * Cfg::BN + Cfg::N0 + (int)rank * Cfg::H1;
        const int kb_end = min(kb_total, (split + 1) * kps);
#pragma unroll 1
        for (int kb = split * kps; kb < kb_end; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          const bool src1 = kb >= geom.kb0;
          if (src1 && !waited) {
            pdl_wait();  // the source-1 operands come from the preceding grid
            waited = true;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
          const int k0 = (src1 ? kb - geom.kb0 : kb) * kBK;
          const int k0a = (src1 && geom.a1_kwrap > 0) ? k0 % geom.a1_kwrap : k0;
          const CUtensorMap* ta = src1 ? &tA1 : &tA0;
          const CUtensorMap* tb = src1 ? &tB1 : &tB0;
          if (!Cfg::A_MN) {
            tma_load_2d_pair(sa, ta, fb, k0a, m0);
          } else {
            tma_load_2d_pair(sa, ta, fb, m0, k0a);
            tma_load_2d_pair(sa + 8192, ta, fb, m0 + 64, k0a);
          }
#pragma unroll
          for (int j = 0; j < Cfg::B0_LOADS; ++j) {
            if (!Cfg::B_MN)
              tma_load_2d_pair(sb + j * Cfg::B_BOX * 128, tb, fb, k0, nb0 + j * Cfg::B_BOX);
            else
              tma_load_2d_pair(sb + j * 8192, tb, fb, nb0 + j * 64, k0);
          }
#pragma unroll
          for (int j = 0; j < Cfg::B1_LOADS; ++j) {
            if (!Cfg::B_MN)
              tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * Cfg::B_BOX * 128, tb, fb, k0, nb1 + j * Cfg::B_BOX);
            else
              tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * 8192, tb, fb, nb1 + j * 64, k0);
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
      int it = 0, j = 0;
      bool ok = true;
#pragma unroll 1
      for (int item = pair; item < items && ok; item += npairs, ++j) {
        const int t = item / splits, split = item - t * splits;
        const int b = j % NACC;
        const uint32_t uph = (uint32_t)(j / NACC) & 1u;
        if (!mbar_wait(&acce[b], uph ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)b * ACC_COLS;
        const int kb_begin = split * kps;
        const int kb_end = min(kb_total, kb_begin + kps);
        (void)t;
#pragma unroll 1
        for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
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
            const uint32_t acc = (kb > kb_begin || kk > 0) ? 1u : 0u;
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
    const int q = warp & 3;
    const int row = q * 32 + lane;
    typename Epi::RowState st{};
    if (defer) pdl_wait();  // before the epilogue reads or writes anything
    int j = 0;
#pragma unroll 1
    for (int item = pair; item < items; item += npairs, ++j) {
      const int t = item / splits, split = item - t * splits;
      const int b = j % NACC;
      const uint32_t uph = (uint32_t)(j / NACC) & 1u;
      if (!mbar_wait(&accf[b], uph)) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, m_tiles, n_tiles, tm, tn);
      const int kb_begin = split * kps;
      EpiCtx c;
      c.taddr = tmem + (uint32_t)b * ACC_COLS + ((uint32_t)(q * 32) << 16);
      c.row = row;
      c.m = tm * 2 * kBM + (int)rank * kBM + row;
      c.n0 = tn * Cfg::BN;
      c.split = split;
      c.has_acc = min(kb_total, kb_begin + kps) > kb_begin;
      c.stage_smem = epi_smem;
      c.stage_bytes = EPI_BYTES;
      c.aux_bar = nullptr;
      c.tA1 = &tA1;
      c.refill_first = 0;
      c.ring_stages = 0;
      c.stage_stride = 0;
      c.tile_id = t;
      c.splits = splits;
      c.flag = nullptr;
      Epi::template run<Cfg::BN>(ep, st, c, geom);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acce[b]), 0));
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

// ------------------------------------------------------------------ CTA-pair split-K variant
//
// One 256 x BN output tile (and one K split, blockIdx.z) per CTA pair, not
// persistent: the pair-tile operand rate of the kernel above, with the 1-CTA
// kernel's epilogue interface (a single accumulator, an idle stage ring and an
// aux barrier after the main loop, split bookkeeping). Epilogues that read the
// A stages (kReadsA: the norm's sum of squares over W0 rows) cannot wait on
// the stages' full barrier, which lives in the leader CTA only; instead the
// leader's MMA thread commits each stage to a "consumed" barrier in both CTAs
// (the stage's data has been read by the tensor cores, so it is in shared
// memory), each CTA's epilogue warps read their own 128 A rows there, and the
// stage returns to that CTA's producer when its four epilogue warps have
// arrived on its empty barrier.

template <class Cfg, class Epi>
struct PairSplitLayout {
  static constexpr int STAGES_RAW = kSmemBudget / Cfg::STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "stages");
  static constexpr int SMEM_BYTES = STAGES * Cfg::STAGE_BYTES + Cfg::BAR_BYTES + 1024;
};

template <class Cfg, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_sm100_pair_split_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                                 const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
                                 const GemmGeom geom, const __grid_constant__ typename Epi::Params ep) {
  constexpr int STAGES = PairSplitLayout<Cfg, Epi>::STAGES;
  constexpr bool READS_A = Epi::kReadsA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* cons = empty + STAGES;  // [STAGES], used when READS_A
  uint64_t* accf = cons + STAGES;
  uint64_t* aux = accf + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux + 1);
  static_assert((3 * 8 + 2) * 8 + 8 <= Cfg::BAR_BYTES, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int n_tiles = (geom.N + Cfg::BN - 1) / Cfg::BN;
  const int t = blockIdx.x >> 1;
  const int tm = t / n_tiles, tn = t - tm * n_tiles;
  const int split = blockIdx.z;
  const int kb_total = geom.kb0 + geom.kb1;
  const int kb_begin = split * geom.kb_per_split;
  const int kb_end = min(kb_total, kb_begin + geom.kb_per_split);
  const int nkb = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], READS_A ? 4 : 1);
      mbar_init(&cons[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(aux, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tA0);
    prefetch_tmap(&tB0);
    if (geom.kb1 > 0) {
      prefetch_tmap(&tA1);
      prefetch_tmap(&tB1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::ACC_COLS);  // one accumulator: one tile per pair
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  const bool defer = geom.defer_wait_src1 != 0;
  if (!defer) pdl_wait();

  const int m0 = tm * 2 * kBM + (int)rank * kBM;
  if (warp == 0) {
    if (lane == 0) {
      const int nb0 = tn * Cfg::BN + (int)rank * Cfg::H0;
      const int nb1 = tn * Cfg::BN + Cfg::N0 + (int)rank * Cfg::H1;
      bool waited = !defer;
      bool ok = true;
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((uint32_t)(i / STAGES) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
        uint8_t* sb = sa + Cfg::A_BYTES;
        const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
        const int kb = kb_begin + i;
        const bool src1 = kb >= geom.kb0;
        if (src1 && !waited) {
          pdl_wait();  // the source-1 operands come from the preceding grid
          waited = true;
        }
        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
        const int k0 = (src1 ? kb - geom.kb0 : kb) * kBK;
        const int k0a = (src1 && geom.a1_kwrap > 0) ? k0 % geom.a1_kwrap : k0;
        const CUtensorMap* ta = src1 ? &tA1 : &tA0;
        const CUtensorMap* tb = src1 ? &tB1 : &tB0;
        if (!Cfg::A_MN) {
          tma_load_2d_pair(sa, ta, fb, k0a, m0);
        } else {
          tma_load_2d_pair(sa, ta, fb, m0, k0a);
          tma_load_2d_pair(sa + 8192, ta, fb, m0 + 64, k0a);
        }
#pragma unroll
        for (int j = 0; j < Cfg::B0_LOADS; ++j) {
          if (!Cfg::B_MN)
            tma_load_2d_pair(sb + j * Cfg::B_BOX * 128, tb, fb, k0, nb0 + j * Cfg::B_BOX);
          else
            tma_load_2d_pair(sb + j * 8192, tb, fb, nb0 + j * 64, k0);
        }
#pragma unroll
        for (int j = 0; j < Cfg::B1_LOADS; ++j) {
          if (!Cfg::B_MN)
            tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * Cfg::B_BOX * 128, tb, fb, k0, nb1 + j * Cfg::B_BOX);
          else
            tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * 8192, tb, fb, nb1 + j * 64, k0);
        }
      }
      if constexpr (Epi::kRefillA1) {
        // The epilogue's rows of the A source-1 operand (this CTA's 128 rows, 64-column
        // slabs of 16 KB), loaded into the ring stages as the last k-blocks release
        // them, so they arrive while the final MMAs still run.
        constexpr int kSps = Cfg::STAGE_BYTES / 16384;
        static_assert(kSps >= 1 && (Cfg::BN / 64 + kSps - 1) / kSps <= STAGES, "refill fits the ring");
        const int slabs = Epi::refill_slabs(ep);
        if (ok && slabs > 0) {
          mbar_arrive_expect_tx(aux, (uint32_t)slabs * 16384u);
          for (int sl = 0; sl < slabs; ++sl) {
            const int u = nkb + sl / kSps;
            const int s = u % STAGES;
            if (sl % kSps == 0 && !mbar_wait(&empty[s], ((uint32_t)(u / STAGES) & 1u) ^ 1u)) break;
            tma_load_2d(smem + s * Cfg::STAGE_BYTES + (sl % kSps) * 16384, &tA1, aux, sl * 64, m0);
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
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], (uint32_t)(i / STAGES) & 1u)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sa + kk * a_kstep, a_lbo, 1024u);
          const uint64_t bd0 = sdesc_sw128(sb + kk * b_kstep, b_lbo, 1024u);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_bf16_pair(tmem, ad, bd0, idesc0, acc);
          if (Cfg::N1 > 0) {
            const uint64_t bd1 = sdesc_sw128(sb + Cfg::B1_OFFSET + kk * b_kstep, b_lbo, 1024u);
            umma_bf16_pair(tmem + (uint32_t)Cfg::N0, ad, bd1, idesc1, acc);
          }
        }
        umma_commit_pair(READS_A ? &cons[s] : &empty[s], 0x3);
      }
      umma_commit_pair(accf, 0x3);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    typename Epi::RowState st{};
    if (READS_A) {
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&cons[s], (uint32_t)(i / STAGES) & 1u)) break;
        Epi::on_a_stage(ep, st, smem + s * Cfg::STAGE_BYTES + row * 128, kb_begin + i >= geom.kb0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    mbar_wait(accf, 0);
    tc_fence_after();
    if (defer) pdl_wait();  // before the epilogue writes anything
    EpiCtx c;
    c.taddr = tmem + ((uint32_t)(q * 32) << 16);
    c.row = row;
    c.m = m0 + row;
    c.n0 = tn * Cfg::BN;
    c.split = split;
    c.has_acc = nkb > 0;
    c.stage_smem = smem;
    c.stage_bytes = STAGES * Cfg::STAGE_BYTES;
    c.aux_bar = aux;
    c.tA1 = &tA1;
    c.refill_first = nkb;
    c.ring_stages = STAGES;
    c.stage_stride = Cfg::STAGE_BYTES;
    c.tile_id = (tm * 2 + (int)rank) * n_tiles + tn;
    c.splits = (int)gridDim.z;
    c.flag = tmem_slot + 1;
    Epi::template run<Cfg::BN>(ep, st, c, geom);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::ACC_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair cluster split-K variant
//
// For GEMMs whose output tiles are too few to fill the GPU (the narrow rank-r
// GEMMs with N = r and a long K, and the base GEMMs of small token batches): a
// cluster of 2 * CS CTAs, i.e. CS CTA pairs (1 to 4, or 8: 16 CTAs, a cluster
// size B200 allows as non-portable), computes one 256 x BN output
// tile, pair z (cluster ranks 2z and 2z + 1) taking the z-th K range. K may
// come from two sources back to back, as in the other kernels. Each pair runs
// the pair kernels' main loop (its leader is rank 2z; commits go to the pair's
// two CTAs). The accumulators are then reduced inside the cluster, CW columns
// at a time: every CTA drains its 128 TMEM rows into its own shared memory
// (the idle stage ring), and after a cluster barrier CTA (z, q) sums rows
// [z * 128 / CS, (z + 1) * 128 / CS) of half q over the cluster's CS CTAs of
// that half, always in split order, by reading their buffers through
// distributed shared memory, and stores them: bf16 alpha * acc (row-major, or
// transposed out[n][m]), or the forward's compose y = acc + gm1[n] acc with
// pre = acc. No fp32 partials reach global memory and the result does not
// depend on timing.

struct ClusterOut {
  __nv_bfloat16* out;  // alpha * acc, or y in compose mode
  __nv_bfloat16* pre;  // compose mode: acc rounded (may be null)
  const float* gm1;    // compose mode: g - 1 per output column
  long long ldo;       // row length of out (elements)
  float alpha;
  int transpose;       // 0: out[m][n]; 1: out[n][m] (not with compose)
  int compose;
};

template <class Cfg>
struct PairClusterLayout {
  static constexpr int STAGES_RAW = kSmemBudget / Cfg::STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "stages");
  // Columns reduced per round: the whole tile when its fp32 rows fit the ring, else 256.
  static constexpr bool ONE_ROUND = 128 * (Cfg::BN + 4) * 4 <= STAGES * Cfg::STAGE_BYTES;
  static constexpr int CW = ONE_ROUND ? Cfg::BN : 256;
  static constexpr int RS = CW + 4;  // fp32 row stride of the reduction buffer
  static_assert(Cfg::BN % CW == 0 || Cfg::BN == 384, "whole rounds");
  static_assert(128 * RS * 4 <= STAGES * Cfg::STAGE_BYTES, "reduction buffer fits the ring");
  static constexpr int SMEM_BYTES = STAGES * Cfg::STAGE_BYTES + Cfg::BAR_BYTES + 1024;
};

template <class Cfg, int CS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_sm100_pair_cluster_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                                   const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
                                   const GemmGeom geom, const ClusterOut o) {
  static_assert((CS >= 1 && CS <= 4) || CS == 8, "pairs per cluster");
  using L = PairClusterLayout<Cfg>;
  constexpr int STAGES = L::STAGES;
  constexpr int CW = L::CW;
  constexpr int RS = L::RS;
  // Rows of its half each CTA reduces: ROWS (a multiple of 8), the last CTA the rest.
  constexpr int ROWS = 8 * ((16 + CS - 1) / CS);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  float* red = reinterpret_cast<float*>(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t q = crank & 1u;              // half of the 256-row tile
  const int z = (int)(crank >> 1);            // K split
  const uint32_t leader = crank & ~1u;
  const uint16_t pair_mask = (uint16_t)(3u << leader);
  const int n_tiles = (geom.N + Cfg::BN - 1) / Cfg::BN;
  const int t = blockIdx.x / (2 * CS);
  const int tm = t / n_tiles, tn = t - tm * n_tiles;
  const int kb_total = geom.kb0 + geom.kb1;
  const int kb_begin = z * geom.kb_per_split;
  const int kb_end = min(kb_total, kb_begin + geom.kb_per_split);
  const int nkb = kb_end > kb_begin ? kb_end - kb_begin : 0;
  const int m0 = tm * 2 * kBM + (int)q * kBM;

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tA0);
    prefetch_tmap(&tB0);
    if (geom.kb1 > 0) {
      prefetch_tmap(&tA1);
      prefetch_tmap(&tB1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::ACC_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_handshake(geom);
  const bool defer = geom.defer_wait_src1 != 0 && !geom.wait_then_trigger;

  if (warp == 0) {
    if (lane == 0) {
      const int nb0 = tn * Cfg::BN + (int)q * Cfg::H0;
      const int nb1 = tn * Cfg::BN + Cfg::N0 + (int)q * Cfg::H1;
      bool waited = !defer;
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((uint32_t)(i / STAGES) & 1u) ^ 1u)) break;
        uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
        uint8_t* sb = sa + Cfg::A_BYTES;
        const uint32_t fb = mapa_shared(smem_u32(&full[s]), leader);
        const int kb = kb_begin + i;
        const bool src1 = kb >= geom.kb0;
        if (src1 && !waited) {
          pdl_wait();  // the source-1 operands come from the preceding grid
          waited = true;
        }
        if (q == 0) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
        const int k0 = (src1 ? kb - geom.kb0 : kb) * kBK;
        const CUtensorMap* ta = src1 ? &tA1 : &tA0;
        const CUtensorMap* tb = src1 ? &tB1 : &tB0;
        if (!Cfg::A_MN) {
          tma_load_2d_pair(sa, ta, fb, k0, m0);
        } else {
          tma_load_2d_pair(sa, ta, fb, m0, k0);
          tma_load_2d_pair(sa + 8192, ta, fb, m0 + 64, k0);
        }
#pragma unroll
        for (int j = 0; j < Cfg::B0_LOADS; ++j) {
          if (!Cfg::B_MN)
            tma_load_2d_pair(sb + j * Cfg::B_BOX * 128, tb, fb, k0, nb0 + j * Cfg::B_BOX);
          else
            tma_load_2d_pair(sb + j * 8192, tb, fb, nb0 + j * 64, k0);
        }
#pragma unroll
        for (int j = 0; j < Cfg::B1_LOADS; ++j) {
          if (!Cfg::B_MN)
            tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * Cfg::B_BOX * 128, tb, fb, k0, nb1 + j * Cfg::B_BOX);
          else
            tma_load_2d_pair(sb + Cfg::B1_OFFSET + j * 8192, tb, fb, nb1 + j * 64, k0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && q == 0) {
      constexpr uint32_t idesc0 = idesc_bf16_f32(2 * kBM, Cfg::N0, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t idesc1 = idesc_bf16_f32(2 * kBM, Cfg::N1 > 0 ? Cfg::N1 : 16, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t a_kstep = Cfg::A_MN ? 2048u : 32u;
      constexpr uint32_t b_kstep = Cfg::B_MN ? 2048u : 32u;
      constexpr uint32_t a_lbo = Cfg::A_MN ? 8192u : 16u;
      constexpr uint32_t b_lbo = Cfg::B_MN ? 8192u : 16u;
#pragma unroll 1
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], (uint32_t)(i / STAGES) & 1u)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sa + kk * a_kstep, a_lbo, 1024u);
          const uint64_t bd0 = sdesc_sw128(sb + kk * b_kstep, b_lbo, 1024u);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_bf16_pair(tmem, ad, bd0, idesc0, acc);
          if (Cfg::N1 > 0) {
            const uint64_t bd1 = sdesc_sw128(sb + Cfg::B1_OFFSET + kk * b_kstep, b_lbo, 1024u);
            umma_bf16_pair(tmem + (uint32_t)Cfg::N0, ad, bd1, idesc1, acc);
          }
        }
        umma_commit_pair(&empty[s], pair_mask);
      }
      umma_commit_pair(accf, pair_mask);
    }
    __syncwarp();
  }

  // ---- reduction inside the cluster, CW columns per round
  if (defer) pdl_wait();  // before the reduction reads or writes anything global
  bool acc_ok = true;
  if (warp >= 2) {
    // tcgen05.ld is warp-collective: the whole warp takes the same branch below.
    acc_ok = __all_sync(0xffffffffu, mbar_wait(accf, 0));
    tc_fence_after();
  }
  const int row_lo = min(128, z * ROWS);
  const int rows = min(128, row_lo + ROWS) - row_lo;
#pragma unroll 1
  for (int c0 = 0; c0 < Cfg::BN; c0 += CW) {
    const int cw = min(CW, Cfg::BN - c0);
    if (warp >= 2) {
      const int qq = warp & 3;
      const int row = qq * 32 + lane;
      float* dst = red + row * RS;
      // 128 columns of TMEM in flight per wait.
#pragma unroll 1
      for (int col = 0; col < cw; col += 128) {
        uint32_t v[4][32];
        const int nch = min(4, (cw - col) / 32);
        if (nkb > 0 && acc_ok) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (c < nch) tmem_ld32_async(tmem + ((uint32_t)(qq * 32) << 16) + (uint32_t)(c0 + col + 32 * c), v[c]);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) v[c][i] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c >= nch) break;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + col + 32 * c + i) =
                make_float4(__uint_as_float(v[c][i]), __uint_as_float(v[c][i + 1]), __uint_as_float(v[c][i + 2]),
                            __uint_as_float(v[c][i + 3]));
        }
      }
    }
    tc_fence_before();
    cluster_sync();  // every CTA's round is in its buffer
    // The CS buffers of this half, read through generic pointers, items summed in
    // split order. Consecutive threads read consecutive 16-byte units of a row, so
    // a warp's load is one contiguous 512-byte run of a peer's shared memory: the
    // cluster network moves such runs several times faster than units spread at
    // a stride (measured on B200: about 5 us against 9 us for the 147 KB a CTA
    // reads at r = 384 and three pairs).
    const float* srcs[CS];
#pragma unroll
    for (int zz = 0; zz < CS; ++zz) srcs[zz] = zz == z ? red : dsmem_ptr(red, (uint32_t)(2 * zz) + q);  // own: local
    if (!o.transpose) {
      // item = (row, 4 columns): out[m][n .. n + 3]. kU items per thread per batch: all
      // their loads are issued before any is summed (kU * CS reads in flight).
      constexpr int kU = CS > 4 ? 2 : 4;
      const int per_row = cw / 4;
      const int n_items = rows * per_row;
#pragma unroll 1
      for (int it0 = threadIdx.x; it0 < n_items; it0 += kGemmThreads * kU) {
        float4 x[kU][CS];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int it = it0 + u * kGemmThreads;
          if (it < n_items) {
            const int off = (row_lo + it / per_row) * RS + (it % per_row) * 4;
#pragma unroll
            for (int zz = 0; zz < CS; ++zz) x[u][zz] = *reinterpret_cast<const float4*>(srcs[zz] + off);
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int it = it0 + u * kGemmThreads;
          if (it >= n_items) break;
          const int lr = row_lo + it / per_row;
          const int lc = (it % per_row) * 4;
          float4 a = x[u][0];
#pragma unroll
          for (int zz = 1; zz < CS; ++zz) {
            a.x += x[u][zz].x;
            a.y += x[u][zz].y;
            a.z += x[u][zz].z;
            a.w += x[u][zz].w;
          }
          const int m = m0 + lr;
          const int n = tn * Cfg::BN + c0 + lc;
          if (m < geom.M && n < geom.N) {
            __nv_bfloat16* dst = o.out + (long long)m * o.ldo + n;
            if (o.compose) {
              // y = pre + (g - 1) pre in fp32, rounded once; y is not read again in the step.
              const float4 gm = __ldg(reinterpret_cast<const float4*>(o.gm1 + n));
              store_bf16x4_cs(dst, fmaf(gm.x, a.x, a.x), fmaf(gm.y, a.y, a.y), fmaf(gm.z, a.z, a.z),
                              fmaf(gm.w, a.w, a.w));
              if (o.pre) store_bf16x4(o.pre + (long long)m * o.ldo + n, a.x, a.y, a.z, a.w);
            } else {
              store_bf16x4(dst, o.alpha * a.x, o.alpha * a.y, o.alpha * a.z, o.alpha * a.w);
            }
          }
        }
      }
    } else {
      // item = (4 columns, 8 rows): out[n .. n + 3][m .. m + 7]; the 8 loads of up to four
      // splits are issued before any is summed, the splits added in order.
      constexpr int ZC = CS < 4 ? CS : 4;
      const int quads = cw / 4;
      const int n_items = (rows / 8) * quads;
#pragma unroll 1
      for (int it = threadIdx.x; it < n_items; it += kGemmThreads) {
        const int lc = (it % quads) * 4;
        const int lr = row_lo + (it / quads) * 8;
        float4 v[8];
#pragma unroll
        for (int zz0 = 0; zz0 < CS; zz0 += ZC) {
          float4 x[ZC][8];
#pragma unroll
          for (int zz = 0; zz < ZC; ++zz)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              x[zz][i] = *reinterpret_cast<const float4*>(srcs[zz0 + zz] + (lr + i) * RS + lc);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int zz = 0; zz < ZC; ++zz) {
              if (zz0 + zz == 0) {
                v[i] = x[0][i];
              } else {
                v[i].x += x[zz][i].x;
                v[i].y += x[zz][i].y;
                v[i].z += x[zz][i].z;
                v[i].w += x[zz][i].w;
              }
            }
          }
        }
        float a[4][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          a[0][i] = o.alpha * v[i].x;
          a[1][i] = o.alpha * v[i].y;
          a[2][i] = o.alpha * v[i].z;
          a[3][i] = o.alpha * v[i].w;
        }
        const int m = m0 + lr;
        const int n = tn * Cfg::BN + c0 + lc;
        if (m < geom.M && n < geom.N) {
#pragma unroll
          for (int j = 0; j < 4; ++j) store_bf16x8(o.out + (long long)(n + j) * o.ldo + m, a[j]);
        }
      }
    }
    cluster_sync();  // the buffers are read before the next round overwrites them (or the CTAs leave)
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::ACC_COLS);
  }
}

// ------------------------------------------------------------------ epilogues

struct NoRowState {};

// out[m, n] = alpha * acc  (or out[n, m] when transposed), bf16.
struct EpiStoreBF16 {
  struct Params {
    __nv_bfloat16* out;
    long long ldo;
    float alpha;
    int transpose;
  };
  using RowState = NoRowState;
  static constexpr bool kReadsA = false;
  static constexpr bool kRefillA1 = false;
  static constexpr int kStageOutBytes = 0;
  __device__ static void on_a_stage(const Params&, RowState&, const uint8_t*, bool) {}
  template <int BN>
  __device__ static void run(const Params& p, RowState&, const EpiCtx& c, const GemmGeom& g) {
    const bool row_ok = c.m < g.M;
    for_each_acc_chunk<BN>(c, [&](int col, float* v) {
      const int n = c.n0 + col;
      if (!row_ok) return;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= p.alpha;
      // A 16-wide tile is visited as a zero-padded 32-column chunk: stores stop
      // at the tile's own width as well as at N.
      if (!p.transpose) {
        __nv_bfloat16* dst = p.out + (long long)c.m * p.ldo + n;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col + 8 * j < BN && n + 8 * j < g.N) store_bf16x8(dst + 8 * j, v + 8 * j);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col + i < BN && n + i < g.N) p.out[(long long)(n + i) * p.ldo + c.m] = __float2bfloat16_rn(v[i]);
      }
    });
  }
};

// part[split][m][n] = acc (fp32), row length ldp; summed later in split order.
struct EpiPartialF32 {
  struct Params {
    float* part;
    long long ldp;
    long long split_stride;
  };
  using RowState = NoRowState;
  static constexpr bool kReadsA = false;
  static constexpr bool kRefillA1 = false;
  static constexpr int kStageOutBytes = 0;
  __device__ static void on_a_stage(const Params&, RowState&, const uint8_t*, bool) {}
  template <int BN>
  __device__ static void run(const Params& p, RowState&, const EpiCtx& c, const GemmGeom& g) {
    const bool row_ok = c.m < g.M;
    float* base = p.part + (long long)c.split * p.split_stride + (long long)c.m * p.ldp;
    for_each_acc_chunk<BN>(c, [&](int col, float* v) {
      const int n = c.n0 + col;
      if (!row_ok) return;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (col + 4 * j < BN && n + 4 * j < g.N)
          *reinterpret_cast<float4*>(base + n + 4 * j) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    });
  }
};

// fp32 partial tiles written by TMA: each epilogue warp stages its 32 rows x
// 32 columns (128 bytes per row, 128-byte swizzle) in one of two 4 KB buffers
// of its own and stores them with a 3-D bulk tensor store over
// [split][row][column], which clips rows past M and columns past N.
struct EpiPartialTMA {
  struct Params {
    CUtensorMap map;  // fp32 {N, M, splits}, box {32, 32, 1}, 128-byte swizzle
  };
  using RowState = NoRowState;
  static constexpr bool kReadsA = false;
  static constexpr bool kRefillA1 = false;
  static constexpr int kStageOutBytes = 4 * 2 * 4096;
  __device__ static void on_a_stage(const Params&, RowState&, const uint8_t*, bool) {}
  template <int BN>
  __device__ static void run(const Params& p, RowState&, const EpiCtx& c, const GemmGeom& g) {
    static_assert(BN % 32 == 0, "whole 32-column chunks");
    const int q = c.row >> 5;
    const int lane = c.row & 31;
    uint8_t* bufs = c.stage_smem + q * 8192;
    const int row0 = c.m - lane;
    int chunk = 0;
    for_each_acc_chunk<BN>(c, [&](int col, float* v) {
      uint8_t* buf = bufs + (chunk & 1) * 4096;
      if (chunk >= 2) {
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && c.n0 + col < g.N && row0 < g.M) {
        tma_store_3d(&p.map, buf, c.n0 + col, row0, c.split);
        bulk_commit();
      }
      ++chunk;
    });
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

// ------------------------------------------------------------------ K-split finish
//
// With the K loop split over blockIdx.z, an epilogue whose per-tile result is
// small can finish it in place: every split CTA stores its partial, then
// counts itself in the tile's counter (zeroed before the launch); the CTA that
// completes the count re-reads all partials in split order (so the result does
// not depend on which CTA came last). Called by all 128 epilogue threads after
// their partial stores; true in the CTA that completes the tile.
// Ordering: the barrier orders every epilogue thread's partial stores before
// thread 0's counter update, which releases them at GPU scope (release is
// cumulative over what the barrier ordered before it); in the completing CTA
// the same acq_rel update acquires the other CTAs' released stores, and the
// second barrier passes that on to the threads that read them.
__device__ __forceinline__ bool split_arrive_last(const EpiCtx& c, unsigned int* counters) {
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (c.row == 0) {
    unsigned int old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(counters + c.tile_id) : "memory");
    *c.flag = (old == (unsigned int)(c.splits - 1)) ? 1u : 0u;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  return *reinterpret_cast<volatile uint32_t*>(c.flag) != 0u;
}

}  // namespace dora
