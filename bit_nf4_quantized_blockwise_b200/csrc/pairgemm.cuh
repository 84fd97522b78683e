// pairgemm.cuh - bf16 GEMM with the LoRA term in the accumulator, on SM pairs
// (tcgen05 cta_group::2), for the QLoRA linear layer at many tokens
// (diycv.top walkthrough, "关键公式": Y = X doubleDequant(c1, c2, W)
// + s X L1 L2; "训练" step 5 for dX = dY W'^T + s dY L2^T L1^T).
//
// pair_gemm_kernel computes D = A * W'(op) + A_ext * B_ext with W' already
// dequantized to bf16 in memory (one pass of nf4_dequant_kernel per call):
// at M >= 1024 tokens dequantizing every weight tile once and streaming it as
// a plain bf16 operand beats re-expanding it in each 256-row tile of the fused
// kernel, whose expansion (byte-permute lookups) bounds it below the tensor
// core's rate.
//   - Pair tile 256 x 256: each CTA of a two-CTA cluster loads 128 rows of A
//     and 128 rows (N) of B per 128-deep stage by TMA; one
//     tcgen05.mma.cta_group::2 of M = N = 256 issued by the even CTA reads both
//     halves, and each CTA's tensor memory receives its own 128 rows of D.
//   - Persistent: pair c takes work items c, c + C, ... (tiles in bands of 8
//     output-column tiles, columns fastest inside a band); two TMEM
//     accumulators per CTA let the drain of one tile overlap the next tile's
//     main loop.  When the last round would hold fewer tiles than pairs,
//     those tiles are split along K into up to four parts that run first;
//     their fp32 partials are summed in part order by the warp that finishes
//     a tile's last part.
//   - Forward: W'^T [o][h] is the K-major B (rows = outputs).  Backward: the
//     same array is the MN-major B of dX = dY W'^T (K = o rows, N = h), loaded
//     as 64-wide N atoms of 128 K rows.  One 2-D tensor map (box 64 x 128,
//     128-byte swizzle) serves both.
//   - LoRA stages: A_ext = [s T_hi | s T_lo], B_ext = [L2; L2] (backward:
//     [s U_hi | s U_lo], [L1; L1]), both K-major, appended to the K loop.
// Warp roles (256 threads per CTA): warp 0 lane 0 issues the TMA loads, whose
// bytes (both CTAs') complete on the even CTA's barrier; warp 1 allocates TMEM
// and, in the even CTA, lane 0 issues the MMAs; warps 4..7 drain TMEM.
#pragma once

#include "common.cuh"

namespace qlora {

// ------------------------------------------------------------------ cluster helpers

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_index_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// Every thread of both CTAs: release this CTA's prior writes, wait for all.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Shared::cluster address of the object at `p` in the CTA of the given rank.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by its shared::cluster address (either CTA).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// Arrive on the even CTA's copy of `bar`: a local arrive in the even CTA.
__device__ __forceinline__ void mbar_arrive_even(uint64_t* bar, uint32_t rank) {
  if (rank == 0)
    mbar_arrive(bar);
  else
    mbar_arrive_remote(cluster_addr(bar, 0));
}

// try_wait with a suspend-time hint: a waiting warp sleeps in hardware until
// the phase completes (or the hint elapses) instead of polling.  kCluster:
// acquire at cluster scope, for barriers the other CTA of the pair arrives on.
template <bool kCluster>
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity) {
  constexpr uint32_t kHintNs = 1000000;
  uint32_t done;
  if (kCluster)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kHintNs)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kHintNs)
        : "memory");
  return done != 0;
}

// Bounded wait (gives up after kWaitLimitNs like mbar_wait, recording the
// site's tag) built on the suspending try_wait.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_idle(uint64_t* bar, uint32_t parity, int tag) {
  if (mbar_try_wait_hint<kCluster>(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_hint<kCluster>(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_status, kStatusTimeout);
      atomicOr(&g_wait_tags, 1u << (tag & 31));
      return false;
    }
  }
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar` is a shared::cluster address).
// No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                                 int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// TMEM allocation shared by the pair: the same warp of both CTAs executes it
// with the same shared-memory destination.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A * B over the pair: A rows 0..127 / 128..255 and B rows (N)
// 0..127 / 128..255 come from the even / odd CTA's shared memory at the same
// descriptor addresses; each CTA's TMEM holds its 128 rows of D.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on the mbarrier at `bar`'s offset in every CTA of `cta_mask` once
// all previously issued tcgen05.mma of this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ====================================================================== pair-tile bf16 GEMM

constexpr int PG_BM = 256;                     // rows of D per pair tile (128 per CTA)
constexpr int PG_BN = 256;                     // cols of D per pair tile (B: 128 rows per CTA)
constexpr int PG_BK = 128;                     // reduction depth of a stage
constexpr int PG_STAGES = 3;
constexpr int PG_THREADS = 256;
constexpr int PG_ATOM_BYTES = 128 * 64 * 2;    // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr int PG_OPND_BYTES = 2 * PG_ATOM_BYTES;  // one CTA's A or B per stage: 32 KB
constexpr int PG_ACC_COLS = 256;               // TMEM columns of one accumulator
constexpr int PG_BAR_BYTES = 128;              // 10 mbarriers and the TMEM address
constexpr int PG_BAND = 8;                     // output-column tiles per band of the tile order
constexpr int PG_SMEM_BYTES = 2 * PG_STAGES * PG_OPND_BYTES + PG_BAR_BYTES + 1024;
static_assert((2 * PG_STAGES + 4) * 8 + 4 <= PG_BAR_BYTES, "barrier area");
static_assert(PG_STAGES == 3, "the MMA issuer selects among three slot descriptors");

// Wait-site tags (bit index in g_wait_tags).
constexpr int kTagPgEmpty = 8, kTagPgFull = 9, kTagPgTFull = 13, kTagPgTEmpty = 14;

struct PairGemmParams {
  int M;              // rows of D (tokens)
  int N;              // cols of D
  int k_main_stages;  // ceil(reduction over W' / 128)
  int k_ext_stages;   // LoRA extension length / 128
  int n_tiles;        // pair tiles along N
  int units;          // pair tiles in all
  int full_units;     // tiles computed whole; the rest (fewer than the pairs) are split along K
  int split;          // K parts of each split tile (1: none)
  float* partial;     // [tail tiles * split][256][256] fp32 partial accumulators
  unsigned* counters; // [tail tiles][2 CTAs][4 warps] arrivals, zero at launch
  void* out;
  int out_bf16;
  int64_t ld_out;
};

// Shared-memory layout per CTA and stage: A and B each as two 16 KB columns
// of the 128-byte swizzle (K 0..63, K 64..127) of 128 rows; the MN-major B of
// the backward as two 64-wide N atoms of 128 K rows each.
template <bool kBwd>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PG_THREADS, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmAe, const __grid_constant__ CUtensorMap tmBe,
                     const __grid_constant__ PairGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sA = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sB = sA + PG_STAGES * PG_OPND_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + PG_STAGES * PG_OPND_BYTES);
  uint64_t* full = bars;                 // even CTA: TMA bytes of both CTAs (+ its producer)
  uint64_t* empty = full + PG_STAGES;    // each CTA: the MMA's commit
  uint64_t* tfull = empty + PG_STAGES;   // each CTA: accumulator complete
  uint64_t* tempty = tfull + 2;          // even CTA: the 8 epilogue warps of the pair
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_index_x());
  const int npairs = static_cast<int>(cluster_count_x());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KM = p.k_main_stages;
  const int S = KM + p.k_ext_stages;
  // Tile u walks bands of PG_BAND output-column tiles: inside a band the
  // column index runs fastest, then the row index, so the pairs working at
  // one time share about PG_BAND panels of B and npairs / PG_BAND panels of A
  // in L2.
  const int m_tiles = p.units / p.n_tiles;
  auto tile_of = [&](int u, int& m0, int& n0) {
    const int band = u / (PG_BAND * m_tiles);
    const int r = u - band * PG_BAND * m_tiles;
    const int width = min(PG_BAND, p.n_tiles - band * PG_BAND);
    m0 = (r / width) * PG_BM;
    n0 = (band * PG_BAND + r % width) * PG_BN;
  };
  // Work items: first the K parts of the tiles from full_units on (part j of
  // a split tile covers stages [j S / split, (j + 1) S / split)), then tiles
  // 0 .. full_units - 1 whole.  Splitting the tiles of a short last round
  // balances the pairs; running the parts first hides the summation of their
  // partial accumulators behind the whole tiles that follow.  Pair c takes
  // items c, c + C, ...
  const int n_parts = (p.units - p.full_units) * p.split;
  const int n_items = p.full_units + n_parts;
  const int nk = pair < n_items ? (n_items - 1 - pair) / npairs + 1 : 0;  // items of this pair
  struct Item {
    int m0, n0, kbeg, kend;
    int slot;  // index of a split part (-1: a whole tile)
  };
  auto item_of = [&](int k) -> Item {
    const int u = pair + k * npairs;
    Item it;
    if (u >= n_parts) {
      tile_of(u - n_parts, it.m0, it.n0);
      it.kbeg = 0;
      it.kend = S;
      it.slot = -1;
    } else {
      const int part = u % p.split;
      tile_of(p.full_units + u / p.split, it.m0, it.n0);
      it.kbeg = part * S / p.split;
      it.kend = (part + 1) * S / p.split;
      it.slot = u;
    }
    return it;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < PG_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
    tma_prefetch_map(&tmAe);
    tma_prefetch_map(&tmBe);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * PG_ACC_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_barrier();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: per stage this CTA's 128 rows of A and of B
      // (each as two 64-wide boxes); both CTAs' bytes complete on the even CTA's full.
      int G = 0;
      bool ok = true;
      for (int k = 0; k < nk && ok; ++k) {
        const Item it = item_of(k);
        const int m0 = it.m0 + static_cast<int>(rank) * 128;
        const int n0 = it.n0 + static_cast<int>(rank) * 128;
        for (int i = it.kbeg; i < it.kend; ++i, ++G) {
          const int s = G % PG_STAGES;
          if (!mbar_wait_idle(&empty[s], ((G / PG_STAGES) & 1) ^ 1, kTagPgEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = cluster_addr(&full[s], 0);
          uint8_t* a_dst = sA + s * PG_OPND_BYTES;
          uint8_t* b_dst = sB + s * PG_OPND_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 4 * PG_OPND_BYTES);
          if (i < KM) {
            const int k0 = i * PG_BK;
            tma_load_2d_pair(a_dst, &tmA, fb, k0, m0);
            tma_load_2d_pair(a_dst + PG_ATOM_BYTES, &tmA, fb, k0 + 64, m0);
            if (kBwd) {
              // MN-major B: N atoms n0 and n0 + 64 (W'^T columns), K rows k0 .. k0 + 127
              tma_load_2d_pair(b_dst, &tmB, fb, n0, k0);
              tma_load_2d_pair(b_dst + PG_ATOM_BYTES, &tmB, fb, n0 + 64, k0);
            } else {
              tma_load_2d_pair(b_dst, &tmB, fb, k0, n0);
              tma_load_2d_pair(b_dst + PG_ATOM_BYTES, &tmB, fb, k0 + 64, n0);
            }
          } else {
            const int x = (i - KM) * PG_BK;
            tma_load_2d_pair(a_dst, &tmAe, fb, x, m0);
            tma_load_2d_pair(a_dst + PG_ATOM_BYTES, &tmAe, fb, x + 64, m0);
            tma_load_2d_pair(b_dst, &tmBe, fb, x, n0);
            tma_load_2d_pair(b_dst + PG_ATOM_BYTES, &tmBe, fb, x + 64, n0);
          }
        }
      }
      // Leave no copy in flight: the even CTA's last phases count both CTAs' bytes.
      if (rank == 0)
        for (int g = G - PG_STAGES > 0 ? G - PG_STAGES : 0; g < G; ++g)
          mbar_wait_idle(&full[g % PG_STAGES], (g / PG_STAGES) & 1, kTagPgFull);
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      // ---------------- MMA issuer (even CTA)
      const uint32_t idesc_main = idesc_bf16(PG_BM, PG_BN, false, kBwd);
      const uint32_t idesc_ext = idesc_bf16(PG_BM, PG_BN, false, false);
      // Descriptors of each slot's K offset 0; a k16 step adds its byte offset / 16
      // to the start-address field (addresses stay below 256 KB: no carry out).
      uint64_t a_desc0[PG_STAGES], b_desc0[PG_STAGES], bmn_desc0[PG_STAGES];
#pragma unroll
      for (int s = 0; s < PG_STAGES; ++s) {
        a_desc0[s] = sw128_desc(smem_u32(sA + s * PG_OPND_BYTES), 16, 1024);
        b_desc0[s] = sw128_desc(smem_u32(sB + s * PG_OPND_BYTES), 16, 1024);
        bmn_desc0[s] = sw128_desc(smem_u32(sB + s * PG_OPND_BYTES), PG_ATOM_BYTES, 1024);
      }
      int G = 0;
      bool ok = true;
      for (int k = 0; k < nk && ok; ++k) {
        const int b = k & 1;
        if (!mbar_wait_idle<true>(&tempty[b], ((k >> 1) & 1) ^ 1, kTagPgTEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * PG_ACC_COLS);
        const Item it = item_of(k);
        for (int i = it.kbeg; i < it.kend; ++i, ++G) {
          const int s = G % PG_STAGES;
          if (!mbar_wait(&full[s], (G / PG_STAGES) & 1, kTagPgFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool b_mn = kBwd && i < KM;
          const uint64_t ad = s == 0 ? a_desc0[0] : (s == 1 ? a_desc0[1] : a_desc0[2]);
          const uint64_t bd = b_mn ? (s == 0 ? bmn_desc0[0] : (s == 1 ? bmn_desc0[1] : bmn_desc0[2]))
                                   : (s == 0 ? b_desc0[0] : (s == 1 ? b_desc0[1] : b_desc0[2]));
          const uint32_t idesc = b_mn ? idesc_main : idesc_ext;
#pragma unroll
          for (int kk = 0; kk < PG_BK / 16; ++kk) {
            const uint32_t k_off = ((kk >> 2) * PG_ATOM_BYTES + (kk & 3) * 32) >> 4;
            const uint64_t adesc = ad + k_off;
            const uint64_t bdesc = bd + (b_mn ? static_cast<uint32_t>(kk * 2048 >> 4) : k_off);
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (i > it.kbeg || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty[s], 0x3);
        }
        if (ok) umma_commit_pair(&tfull[b], 0x3);
      }
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: warp q drains TMEM lanes 32 q .. 32 q + 31 (this CTA's rows)
    const int q = warp & 3;
    auto store_row = [&](int m, int n, const float* v) {
      if (m >= p.M || n >= p.N) return;
      if (p.out_bf16) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + static_cast<int64_t>(m) * p.ld_out + n);
        uint32_t h[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) h[t] = pack_bf16x2(v[2 * t], v[2 * t + 1]);
        __stcs(dst, make_uint4(h[0], h[1], h[2], h[3]));
        __stcs(dst + 1, make_uint4(h[4], h[5], h[6], h[7]));
      } else {
        // streaming stores: the output is not read again here, keep L2 for the operands
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<int64_t>(m) * p.ld_out + n);
#pragma unroll
        for (int t = 0; t < 4; ++t) __stcs(dst + t, make_float4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]));
      }
    };
    for (int k = 0; k < nk; ++k) {
      const int b = k & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_idle(&tfull[b], (k >> 1) & 1, kTagPgTFull))) break;
      tc_fence_after();
      const Item it = item_of(k);
      const int row = static_cast<int>(rank) * 128 + q * 32 + lane;  // row within the pair tile
      const int m = it.m0 + row;
      // a split part goes to its slot of the partial buffer instead of the output
      float* part = it.slot >= 0 ? p.partial + (static_cast<int64_t>(it.slot) * PG_BM + row) * PG_BN : nullptr;
#pragma unroll 1
      for (int c = 0; c < PG_ACC_COLS / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * PG_ACC_COLS + c * 16), r);
        tmem_ld_wait();
        if (c == PG_ACC_COLS / 16 - 1) {
          // the accumulator is in registers: hand it back to the MMA issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_even(&tempty[b], rank);
        }
        if (part) {
          float4* dst = reinterpret_cast<float4*>(part + c * 16);
#pragma unroll
          for (int t = 0; t < 4; ++t)
            dst[t] = make_float4(__uint_as_float(r[4 * t]), __uint_as_float(r[4 * t + 1]),
                                 __uint_as_float(r[4 * t + 2]), __uint_as_float(r[4 * t + 3]));
        } else {
          store_row(m, it.n0 + c * 16, reinterpret_cast<const float*>(r));
        }
      }
      if (part) {
        // The warp that completes the last part of a split tile sums the parts of
        // its 32 rows in part order (the same result whichever part is last) and
        // writes them out.
        __threadfence();
        __syncwarp();
        const int tail = it.slot / p.split;
        unsigned prior = 0;
        if (lane == 0) prior = atomicAdd(&p.counters[(tail * 2 + static_cast<int>(rank)) * 4 + q], 1u);
        prior = __shfl_sync(0xFFFFFFFFu, prior, 0);
        if (prior == static_cast<unsigned>(p.split - 1)) {
          __threadfence();
          const float* first = p.partial + (static_cast<int64_t>(tail) * p.split * PG_BM + row) * PG_BN;
#pragma unroll 1
          for (int c = 0; c < PG_ACC_COLS / 16; ++c) {
            float v[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) v[t] = 0.0f;
            for (int j = 0; j < p.split; ++j) {
              const float4* src = reinterpret_cast<const float4*>(first + static_cast<int64_t>(j) * PG_BM * PG_BN + c * 16);
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float4 a = __ldcg(src + t);
                v[4 * t] += a.x;
                v[4 * t + 1] += a.y;
                v[4 * t + 2] += a.z;
                v[4 * t + 3] += a.w;
              }
            }
            store_row(m, it.n0 + c * 16, v);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_barrier();  // no CTA leaves while the other may still touch its barriers or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * PG_ACC_COLS);
  }
}

}  // namespace qlora
