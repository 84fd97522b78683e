// gemm.cuh - tcgen05 (5th-generation tensor core) GEMMs of the QLoRA linear
// layer (diycv.top walkthrough, "关键公式": Y = X doubleDequant(c1, c2, W)
// + s X L1 L2; "训练" step 5 for the backward products).
//
// qgemm_nf4_kernel : D = A * W'(op) + A_ext * B_ext, W' dequantized on the fly.
//   Forward  (Y  = X  W'   + [sT_hi|sT_lo] [L2;L2]) : W' operand K-major.
//   Backward (dX = dY W'^T + [sU_hi|sU_lo] [L1;L1]^T): W' operand MN-major.
//   Warp roles (384 threads): warp 0 lane 0 issues TMA loads of the A tiles,
//   of the packed codes (a ring 4 stages deep) and of the LoRA tiles; warp 1
//   lane 0 issues tcgen05.mma; warps 4..11 ("expanders") build each block's
//   16-entry bf16 table in registers and write the dequantized tile straight
//   into the swizzled shared-memory layout the tensor core reads; warps 0..3
//   drain TMEM.
//   Tile 256 x 256 x 64: two M=128 MMAs share every dequantized B tile, which
//   halves the dequantization work per flop.
//
// gemm_tma_kernel  : D (+)= A * (B [+ B2]) for the rank-r products
//   T = X L1, U = dY L2^T, dL1 = X^T (sU), dL2^T = dY^T (sT), with split-K
//   over the long reduction and fp32 atomic accumulation.
//
// small_m_fwd_kernel: the forward at M <= 32 tokens (decode), weight-streaming.
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int QLORA_MAX_RANK_DEV = 256;

// ====================================================================== fused NF4 GEMM

constexpr int QG_BM = 256;
constexpr int QG_BN = 256;
constexpr int QG_BK = 64;
constexpr int QG_STAGES = 3;
constexpr int QG_CSTAGES = 4;                // depth of the packed-code ring
constexpr int QG_THREADS = 384;
constexpr int QG_TILE_BYTES = 256 * 64 * 2;  // one A or B stage: 32 KB
constexpr int QG_CODE_BYTES = 256 * 64 / 2;  // one stage of packed codes: 8 KB
constexpr int QG_SMEM_BYTES = 2 * QG_STAGES * QG_TILE_BYTES + QG_CSTAGES * QG_CODE_BYTES + 256 + 1024;

struct QGemmParams {
  int M;                 // rows of D (tokens)
  int N;                 // cols of D
  int k_main_stages;     // reduction length / 64 over the NF4 weight
  int k_ext_stages;      // LoRA extension length / 64
  int blocks_per_row;    // h / 64: 64-blocks per row of the stored W^T[o][h]
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  const float* absmax32;  // single-level constants (no double quantization), or null
  void* out;
  int out_bf16;
  int64_t ld_out;
  float codebook[16];
};

template <bool kBwd>
__global__ void __launch_bounds__(QG_THREADS, 1)
    qgemm_nf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAe,
                     const __grid_constant__ CUtensorMap tmBe, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ QGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sA = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sB = sA + QG_STAGES * QG_TILE_BYTES;
  uint8_t* sC = sB + QG_STAGES * QG_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + QG_CSTAGES * QG_CODE_BYTES);
  uint64_t* full_a = bars;                          // TMA bytes of A (and B on LoRA stages)
  uint64_t* full_b = bars + QG_STAGES;              // 8 expander warps
  uint64_t* empty = bars + 2 * QG_STAGES;           // tcgen05.commit
  uint64_t* cfull = bars + 3 * QG_STAGES;           // TMA bytes of a code stage
  uint64_t* cempty = cfull + QG_CSTAGES;            // 8 expander warps
  uint64_t* accum = cempty + QG_CSTAGES;            // last MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * QG_BN;
  const int m0 = blockIdx.y * QG_BM;
  const int KM = p.k_main_stages;
  const int S = KM + p.k_ext_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QG_STAGES; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&full_b[s], 8);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < QG_CSTAGES; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 8);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmAe);
    tma_prefetch_map(&tmBe);
    tma_prefetch_map(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: the code ring runs up to QG_CSTAGES
      // stages ahead of the expanders, the operand ring QG_STAGES ahead of
      // the MMA.
      int issued = 0, c_issued = 0;
      bool ok = true;
      for (int i = 0; i < S && ok; ++i) {
        while (c_issued < KM && c_issued < i + QG_CSTAGES) {
          const int cs = c_issued % QG_CSTAGES;
          if (!mbar_wait(&cempty[cs], ((c_issued / QG_CSTAGES) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&cfull[cs], QG_CODE_BYTES);
          if (kBwd)
            tma_load_2d(sC + cs * QG_CODE_BYTES, &tmC, &cfull[cs], n0 / 2, c_issued * QG_BK);
          else
            tma_load_2d(sC + cs * QG_CODE_BYTES, &tmC, &cfull[cs], c_issued * (QG_BK / 2), n0);
          ++c_issued;
        }
        if (!ok) break;
        const int s = i % QG_STAGES;
        const uint32_t ph = (i / QG_STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        if (i < KM) {
          mbar_arrive_expect_tx(&full_a[s], QG_TILE_BYTES);
          tma_load_2d(sA + s * QG_TILE_BYTES, &tmA, &full_a[s], i * QG_BK, m0);
        } else {
          const int j = i - KM;
          mbar_arrive_expect_tx(&full_a[s], 2 * QG_TILE_BYTES);
          tma_load_2d(sA + s * QG_TILE_BYTES, &tmAe, &full_a[s], j * QG_BK, m0);
          tma_load_2d(sB + s * QG_TILE_BYTES, &tmBe, &full_a[s], j * QG_BK, n0);
        }
        issued = i + 1;
      }
      // Leave no copy in flight: wait (bounded) for the last loads of each ring.
      for (int i = issued - QG_STAGES > 0 ? issued - QG_STAGES : 0; i < issued; ++i)
        mbar_wait(&full_a[i % QG_STAGES], (i / QG_STAGES) & 1);
      for (int i = c_issued - QG_CSTAGES > 0 ? c_issued - QG_CSTAGES : 0; i < c_issued; ++i)
        mbar_wait(&cfull[i % QG_CSTAGES], (i / QG_CSTAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc_main = idesc_bf16(128, QG_BN, false, kBwd);
      const uint32_t idesc_ext = idesc_bf16(128, QG_BN, false, false);
      bool ok = true;
      for (int i = 0; i < S && ok; ++i) {
        const int s = i % QG_STAGES;
        const uint32_t ph = (i / QG_STAGES) & 1;
        ok = mbar_wait(&full_a[s], ph);
        if (ok && i < KM) ok = mbar_wait(&full_b[s], ph);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * QG_TILE_BYTES);
        const uint32_t b_base = smem_u32(sB + s * QG_TILE_BYTES);
        const bool b_mn = kBwd && i < KM;
#pragma unroll
        for (int kk = 0; kk < QG_BK / 16; ++kk) {
          const uint64_t bdesc = b_mn ? sw128_desc(b_base + kk * 2048, 8192, 1024)
                                      : sw128_desc(b_base + kk * 32, 16, 1024);
#pragma unroll
          for (int hm = 0; hm < 2; ++hm) {
            const uint64_t adesc = sw128_desc(a_base + hm * 16384 + kk * 32, 16, 1024);
            umma_bf16(tmem + hm * QG_BN, adesc, bdesc, b_mn ? idesc_main : idesc_ext,
                      (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else if (warp >= 4) {
    // ---------------- expanders: 256 threads, one 64-block each per stage.
    //   forward : row n0 + e of W^T, block column i  -> K-major B row e;
    //   backward: row 64 i + kr of W^T (kr = e % 64), block column n0 / 64 + a
    //             (a = e / 64) -> MN-major B, K row kr, N atom a.
    // In the backward, the 8 lanes of a quarter-warp take 8 consecutive K rows
    // of one atom, so their swizzled stores (and their reads of the
    // 128-byte-swizzled code tile) hit distinct banks.
    const int e = threadIdx.x - 128;
    const int kr = e & 63;     // backward: K row within the stage
    const int atom = e >> 6;   // backward: 64-wide N atom
    const float mu = p.absmax32 ? 0.0f : __ldg(p.dq_mean);
    float q[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = p.codebook[j];
    const bool in_range = kBwd ? (n0 / 64 + atom < p.blocks_per_row) : (n0 + e < p.N);
    auto block_index = [&](int i) -> int64_t {
      return kBwd ? static_cast<int64_t>(i * 64 + kr) * p.blocks_per_row + (n0 >> 6) + atom
                  : static_cast<int64_t>(n0 + e) * p.blocks_per_row + i;
    };
    // Byte offsets of this thread's two 16-byte code chunks in a code stage:
    // forward rows of 32 bytes (no swizzle); backward rows of 128 bytes with
    // the TMA 128-byte swizzle (16-byte chunk index XOR row % 8).  In the
    // forward, rows e and e + 4 share banks, so the lanes with bit 2 of e set
    // read their second chunk first: each quarter-warp then covers all 32
    // banks once (the two chunks are put back in order after the loads).
    const bool swap_chunks = !kBwd && ((e >> 2) & 1);
    const int code_off0 = kBwd ? kr * 128 + (((2 * atom) ^ (kr & 7)) << 4) : e * 32 + (swap_chunks ? 16 : 0);
    const int code_off1 = kBwd ? kr * 128 + (((2 * atom + 1) ^ (kr & 7)) << 4) : e * 32 + (swap_chunks ? 0 : 16);
    uint32_t boff[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (kBwd) {
        boff[c] = atom * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128 + ((c ^ (kr & 7)) << 4);
      } else {
        boff[c] = (e >> 3) * 1024 + (e & 7) * 128 + ((c ^ (e & 7)) << 4);
      }
    }
    // Block constants ride a register ring kPre stages ahead of the expansion
    // (slot t serves stages t, t + kPre, ...; the stage loop is unrolled by
    // kPre so that every slot index is static and no register copy waits on a
    // load in flight).
    constexpr int kPre = 4;
    uint32_t ec[kPre];
    float sc[kPre];
    auto fetch = [&](int i, uint32_t& e8, float& s32) {
      e8 = 0;
      s32 = 0.0f;
      if (in_range && i < KM) {
        const int64_t blk = block_index(i);
        if (p.absmax32) {
          s32 = __ldg(p.absmax32 + blk);  // the block constant itself
        } else {
          e8 = __ldg(p.absmax_fp8 + blk);
          s32 = __ldg(p.dq_scale + (blk >> 8));
        }
      }
    };
#pragma unroll
    for (int t = 0; t < kPre; ++t) fetch(t, ec[t], sc[t]);
    ConstCache cc;
    bool ok = true;
    for (int i0 = 0; i0 < KM && ok; i0 += kPre) {
#pragma unroll
    for (int t = 0; t < kPre; ++t) {
      const int i = i0 + t;
      if (i >= KM) break;
      const int s = i % QG_STAGES;
      const uint32_t ph = (i / QG_STAGES) & 1;
      const int cs = i % QG_CSTAGES;
      const uint32_t cph = (i / QG_CSTAGES) & 1;
      const uint32_t e_now = ec[t];
      const float s_now = sc[t];
      fetch(i + kPre, ec[t], sc[t]);
      Lut16 L;
      build_lut16(q, in_range ? (p.absmax32 ? s_now : cc.constant(static_cast<uint8_t>(e_now), s_now, mu)) : 0.0f,
                  L);
      if (!mbar_wait(&cfull[cs], cph)) {
        ok = false;
        break;
      }
      const uint8_t* cbase = sC + cs * QG_CODE_BYTES;
      const uint4 r0 = *reinterpret_cast<const uint4*>(cbase + code_off0);
      const uint4 r1 = *reinterpret_cast<const uint4*>(cbase + code_off1);
      const uint4 c0 = swap_chunks ? r1 : r0;
      const uint4 c1 = swap_chunks ? r0 : r1;
      if (!mbar_wait(&empty[s], ph ^ 1)) {
        ok = false;
        break;
      }
      uint8_t* bdst = sB + s * QG_TILE_BYTES;
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(bdst + boff[c]) = lut_lookup8(L, words[c]);
      // The proxy fence orders this thread's generic shared-memory accesses
      // (the code reads above and the tile writes) before the async-proxy
      // accesses that follow the releases: the tensor core reading the tile,
      // and the next TMA load overwriting the code slot.  The code slot is
      // released only here, after its values have been consumed.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full_b[s]);
        mbar_arrive(&cempty[cs]);
      }
    }
    }
  }

  // ---------------- epilogue: warps 0..3 drain TMEM (both M halves)
  if (warp < 4) {
    __syncwarp();
    const bool ok = mbar_wait(accum, 0);
    tc_fence_after();
    if (ok) {
      const int q = warp & 3;
#pragma unroll 1
      for (int hm = 0; hm < 2; ++hm) {
        const int m = m0 + hm * 128 + q * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < QG_BN / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + hm * QG_BN + c * 16, r);
          tmem_ld_wait();
          const int n = n0 + c * 16;
          if (m < p.M && n < p.N) {
            if (p.out_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + static_cast<int64_t>(m) * p.ld_out + n);
              uint32_t h[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) h[t] = pack_bf16x2(__uint_as_float(r[2 * t]), __uint_as_float(r[2 * t + 1]));
              dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
              dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<int64_t>(m) * p.ld_out + n);
#pragma unroll
              for (int t = 0; t < 4; ++t)
                dst[t] = make_float4(__uint_as_float(r[4 * t]), __uint_as_float(r[4 * t + 1]),
                                     __uint_as_float(r[4 * t + 2]), __uint_as_float(r[4 * t + 3]));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ====================================================================== TMA GEMM for rank-r products

constexpr int TG_BM = 128;
constexpr int TG_BK = 64;
constexpr int TG_THREADS = 128;
constexpr int TG_MAX_STAGES = 4;
// ring size cap: two CTAs per SM always fit (these kernels are short, and a
// second wave of one CTA per SM would double their time)
constexpr int TG_SMEM_LIMIT = 110 * 1024;
constexpr int TG_SMEM_LIMIT_ONE = 200 * 1024;  // one CTA per SM (stages above 55 KB)

struct TGemmParams {
  int M;               // valid rows of D
  int N;               // valid cols of D
  int bn;              // tile width along N: 64, 128, 192 or 256
  int k_stages;        // total 64-wide K stages
  int k_per_split;     // stages handled by one blockIdx.z
  int stages;          // pipeline depth
  int hilo;            // accumulate A*B + A*B2
  float* out;
  int64_t ld_out;
  int transpose_out;   // store D[m][n] at out[n * ld + m]
  float alpha;         // D is scaled by alpha before it is added
  uint32_t mask_thr;   // with a nonzero threshold, D[m][n] is also multiplied by the
  uint64_t mask_seed;  // dropout keep bit of element m * mask_ld + n (non-transposed
  int64_t mask_ld;     // output only)
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// A operand: K-major  -> tensor [rows of D][K],   box {64, 128}, one load;
//            MN-major -> tensor [K][rows of D],   box {64, 64}, two loads.
// B operand: K-major  -> tensor [cols of D][K],   box {64, bn}, one load;
//            MN-major -> tensor [K][cols of D],   box {64, 64}, bn/64 loads.
template <bool kAmn, bool kBmn>
__global__ void __launch_bounds__(TG_THREADS, 1)
    gemm_tma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ TGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int a_bytes = TG_BM * TG_BK * 2;
  const int b_bytes = p.bn * TG_BK * 2;
  const int stage_bytes = a_bytes + (p.hilo ? 2 : 1) * b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.stages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + TG_MAX_STAGES;
  uint64_t* accum = bars + 2 * TG_MAX_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * TG_MAX_STAGES + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * TG_BM;
  const int nt0 = blockIdx.y * p.bn;
  const int kz0 = blockIdx.z * p.k_per_split;
  int kz1 = kz0 + p.k_per_split;
  kz1 = kz1 < p.k_stages ? kz1 : p.k_stages;
  const int S = kz1 > kz0 ? kz1 - kz0 : 0;
  const uint32_t tmem_cols = p.bn <= 64 ? 64u : (p.bn <= 128 ? 128u : 256u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0 && S > 0) {
    int issued = 0;
    for (int i = 0; i < S; ++i) {
      const int s = i % p.stages;
      const uint32_t ph = (i / p.stages) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1)) break;
      uint8_t* st = smem + s * stage_bytes;
      const int k = (kz0 + i) * TG_BK;
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      if (kAmn) {
        tma_load_2d(st, &tmA, &full[s], m0, k);
        tma_load_2d(st + 8192, &tmA, &full[s], m0 + 64, k);
      } else {
        tma_load_2d(st, &tmA, &full[s], k, m0);
      }
      for (int h = 0; h < (p.hilo ? 2 : 1); ++h) {
        const CUtensorMap* mb = h ? &tmB2 : &tmB;
        uint8_t* sb = st + a_bytes + h * b_bytes;
        if (kBmn) {
          for (int t = 0; t < p.bn / 64; ++t) tma_load_2d(sb + t * 8192, mb, &full[s], nt0 + 64 * t, k);
        } else {
          tma_load_2d(sb, mb, &full[s], k, nt0);
        }
      }
      issued = i + 1;
    }
    for (int i = issued - p.stages > 0 ? issued - p.stages : 0; i < issued; ++i)
      mbar_wait(&full[i % p.stages], (i / p.stages) & 1);
  } else if (warp == 1 && lane == 0 && S > 0) {
    const uint32_t idesc = idesc_bf16(128, p.bn, kAmn, kBmn);
    for (int i = 0; i < S; ++i) {
      const int s = i % p.stages;
      const uint32_t ph = (i / p.stages) & 1;
      if (!mbar_wait(&full[s], ph)) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * stage_bytes);
#pragma unroll
      for (int kk = 0; kk < TG_BK / 16; ++kk) {
        const uint64_t adesc = kAmn ? sw128_desc(a_base + kk * 2048, 8192, 1024)
                                    : sw128_desc(a_base + kk * 32, 16, 1024);
        for (int h = 0; h < (p.hilo ? 2 : 1); ++h) {
          const uint32_t b_base = a_base + a_bytes + h * b_bytes;
          const uint64_t bdesc = kBmn ? sw128_desc(b_base + kk * 2048, 8192, 1024)
                                      : sw128_desc(b_base + kk * 32, 16, 1024);
          umma_bf16(tmem, adesc, bdesc, idesc, (i > 0 || kk > 0 || h > 0) ? 1u : 0u);
        }
      }
      umma_commit(&empty[s]);
    }
    umma_commit(accum);
  }

  __syncwarp();
  const bool ok = S > 0 && mbar_wait(accum, 0);
  tc_fence_after();
  if (ok) {
    const int m = m0 + warp * 32 + lane;
    for (int c = 0; c < p.bn / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 16, r);
      tmem_ld_wait();
      const int n = nt0 + c * 16;
      if (m < p.M && n < p.N) {
        float v[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) v[t] = p.alpha * __uint_as_float(r[t]);
        if (p.transpose_out) {
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (n + t < p.N) atomicAdd(p.out + static_cast<int64_t>(n + t) * p.ld_out + m, v[t]);
        } else {
          float* row = p.out + static_cast<int64_t>(m) * p.ld_out + n;
#pragma unroll
          for (int t = 0; t < 16; t += 4) {
            if (n + t < p.N) {
              if (p.mask_thr) {
                const uint32_t k = dropout_keep4((static_cast<uint64_t>(m) * p.mask_ld + n + t) >> 2, p.mask_seed,
                                                 p.mask_thr);
#pragma unroll
                for (int j = 0; j < 4; ++j) v[t + j] = (k >> j) & 1u ? v[t + j] : 0.0f;
              }
              red_add_v4(row + t, v[t], v[t + 1], v[t + 2], v[t + 3]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ====================================================================== adapter merge into the bf16 base

// W_m = bf16(W' + s L1 L2), stored like the weight as W_m^T[o][h]: the merge
// into the 16-bit dequantized base that the QLoRA glossary's pitfalls entry
// prescribes (never into the 4-bit codes).  The rank-r product runs on the
// tensor cores: one CTA computes D[n][k] = sum_j L2[j][n] L1[k][j] for a
// 128 (n) x 256 (k) tile with tcgen05 (A = L2^T, MN-major, straight from L2's
// rows; B = L1, K-major), every K stage of the rank loaded up front by TMA.
// The epilogue reads the fp32 tile from tensor memory (thread = row n),
// dequantizes the matching 16 weights per step with the block's register
// table (the same bf16(q c') as the dequant kernel), and stores
// bf16(W' + s D) with one final round-to-nearest-even.
constexpr int MG_BM = 128;
constexpr int MG_BN = 256;
constexpr int MG_THREADS = 256;  // 8 warps: two per tensor-memory lane quadrant in the epilogue
constexpr int MG_A_STAGE = MG_BM * 64 * 2;   // 16 KB: two 64 x 64 MN-major atoms of L2
constexpr int MG_B_STAGE = MG_BN * 64 * 2;   // 32 KB: 256 rows of L1, 64 ranks
// Dynamic shared memory is never below this, so that at most two CTAs share an
// SM and their 256-column accumulators fit its 512 tensor-memory columns.
constexpr int MG_MIN_SMEM = 100 * 1024;

struct MergeParams {
  int o, h;             // W^T[o][h]
  int k_stages;         // ceil(r / 64)
  float s;
  const uint8_t* codes; // [o][h/2]
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  const float* absmax32;  // single-level constants, or null
  uint16_t* out;        // bf16 [o][h]
  float codebook[16];
};

__global__ void __launch_bounds__(MG_THREADS, 1)
    merge_kernel(const __grid_constant__ CUtensorMap tmL2, const __grid_constant__ CUtensorMap tmL1,
                 const __grid_constant__ MergeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + p.k_stages * MG_A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + p.k_stages * MG_B_STAGE);
  uint64_t* full = bars;
  uint64_t* accum = bars + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * MG_BM;
  const int k0 = blockIdx.y * MG_BN;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, MG_BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmL2);
    tma_prefetch_map(&tmL1);
    mbar_arrive_expect_tx(full, static_cast<uint32_t>(p.k_stages * (MG_A_STAGE + MG_B_STAGE)));
    for (int s = 0; s < p.k_stages; ++s) {
      tma_load_2d(sA + s * MG_A_STAGE, &tmL2, full, n0, s * 64);
      tma_load_2d(sA + s * MG_A_STAGE + 8192, &tmL2, full, n0 + 64, s * 64);
      tma_load_2d(sB + s * MG_B_STAGE, &tmL1, full, s * 64, k0);
    }
    // no copy may still be landing when the CTA exits
    mbar_wait(full, 0, 12);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(MG_BM, MG_BN, true, false);
    if (mbar_wait(full, 0, 13)) {
      tc_fence_after();
      for (int s = 0; s < p.k_stages; ++s) {
        const uint32_t a_base = smem_u32(sA + s * MG_A_STAGE);
        const uint32_t b_base = smem_u32(sB + s * MG_B_STAGE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, sw128_desc(a_base + kk * 2048, 8192, 1024), sw128_desc(b_base + kk * 32, 16, 1024), idesc,
                    (s > 0 || kk > 0) ? 1u : 0u);
      }
    }
    umma_commit(accum);
  }

  // ---------------- epilogue: thread = weight row n, 16 columns per step;
  // warps w and w + 4 share lane quadrant w % 4 and take one half of the
  // columns each (two 64-blocks).  The thread's 64 code bytes and its two
  // block constants do not depend on the product, so their loads are issued
  // before the wait and overlap the TMA loads and the MMA.
  const int quad = warp & 3, half = warp >> 2;
  const int n = n0 + quad * 32 + lane;
  const bool row_ok = n < p.o;
  const int64_t row_el = static_cast<int64_t>(n) * p.h;
  const int kh = k0 + half * (MG_BN / 2);
  const int nch = kh < p.h ? min(MG_BN / 32, (p.h - kh) / 16) : 0;  // 16-column chunks in range
  uint4 cw4[4] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                  make_uint4(0u, 0u, 0u, 0u)};
  float craw[2] = {0.0f, 0.0f};   // single-level constant, or the group scale
  uint32_t e8[2] = {0u, 0u};      // FP8 code of the block constant
  if (row_ok) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (2 * i < nch) cw4[i] = __ldg(reinterpret_cast<const uint4*>(p.codes + ((row_el + kh) >> 1)) + i);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (4 * b < nch) {
        const int64_t blk = (row_el + kh) / 64 + b;
        if (p.absmax32) {
          craw[b] = __ldg(p.absmax32 + blk);
        } else {
          e8[b] = __ldg(p.absmax_fp8 + blk);
          craw[b] = __ldg(p.dq_scale + (blk >> 8));
        }
      }
    }
  }
  __syncwarp();
  const bool ok = mbar_wait_sleep(accum, 0, 14);
  tc_fence_after();
  if (ok) {
    float q[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = p.codebook[j];
    const float mu = p.absmax32 ? 0.0f : __ldg(p.dq_mean);
    ConstCache cc;
    Lut16 L;
#pragma unroll
    for (int cl = 0; cl < MG_BN / 32; ++cl) {
      const int c = half * (MG_BN / 32) + cl;
      const int k = k0 + 16 * c;
      if (k >= p.h) break;  // the same k for every lane
      uint32_t d[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 16 * c, d);
      tmem_ld_wait();
      if (!row_ok) continue;
      const int64_t e0 = row_el + k;
      if ((cl & 3) == 0) {
        const int b = cl >> 2;
        const float cp = p.absmax32 ? craw[b] : cc.constant(static_cast<uint8_t>(e8[b]), craw[b], mu);
        build_lut16(q, cp, L);
      }
      const uint4 q4 = cw4[cl >> 1];
      const uint32_t cx = (cl & 1) ? q4.z : q4.x, cy = (cl & 1) ? q4.w : q4.y;
      const uint4 w01 = lut_lookup8(L, cx), w23 = lut_lookup8(L, cy);
      const uint32_t wp[8] = {w01.x, w01.y, w01.z, w01.w, w23.x, w23.y, w23.z, w23.w};
      uint32_t o8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = __fadd_rn(__uint_as_float(wp[i] << 16), __fmul_rn(p.s, __uint_as_float(d[2 * i])));
        const float b = __fadd_rn(__uint_as_float(wp[i] & 0xFFFF0000u), __fmul_rn(p.s, __uint_as_float(d[2 * i + 1])));
        o8[i] = pack_bf16x2(a, b);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out + e0);
      dst[0] = make_uint4(o8[0], o8[1], o8[2], o8[3]);
      dst[1] = make_uint4(o8[4], o8[5], o8[6], o8[7]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, MG_BN);
  }
}

// ====================================================================== small element-wise kernels

// The hi/lo bf16 split of s * T for the LoRA extension, row length 2 * rp:
//   c <  r            : hi = bf16(s * T[m][c])
//   rp <= c < rp + r  : lo = bf16(s * T[m][c - rp] - hi)
//   otherwise         : 0
// s * T is one fp32 rounding; hi + lo carries it to ~2^-17 relative.
// blockIdx.y selects one of two (source, destination) pairs.
struct SplitJob {
  const float* src;    // fp32 [M][r]
  uint16_t* dst;       // bf16 [M][2 rp]
};

__global__ void __launch_bounds__(256) lora_split_kernel(SplitJob j0, SplitJob j1, int64_t M, int r, int rp,
                                                         float s) {
  const SplitJob job = blockIdx.y == 0 ? j0 : j1;
  if (job.src == nullptr) return;
  const int64_t total = M * 2 * rp;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / (2 * rp);
    const int c = static_cast<int>(i - m * 2 * rp);
    const int cc = c < rp ? c : c - rp;
    uint16_t out = 0;
    if (cc < r) {
      const float v = __fmul_rn(s, job.src[m * r + cc]);
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      out = c < rp ? __bfloat16_as_ushort(hi)
                   : __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi))));
    }
    job.dst[i] = out;
  }
}

// Operand packing for the rank-r products and the LoRA extension, plus the
// zeroing of the fp32 accumulators, in one launch:
//   blockIdx.y == 0 : L2x[n][c] = L2[c mod rp][n] for (c mod rp) < r, else 0 (o rows of 2 rp);
//                     32 rows per CTA, transposed through shared memory (skipped if L2x is null);
//   blockIdx.y == 1 : L1x[n][c] = L1[n][c mod rp] for (c mod rp) < r, else 0 (h rows);
//   blockIdx.y == 2 : zero up to four fp32 buffers (lengths multiples of 4,
//                     16-byte aligned).  All accesses are 16-byte vectors.
struct PrepParams {
  const uint16_t* L1;  // [h][r]
  const uint16_t* L2;  // [r][o]
  uint16_t* L1x;       // [h][2 rp]
  uint16_t* L2x;       // [o][2 rp]
  int64_t h, o;
  int r, rp;
  float* zero_ptr[4];
  int64_t zero_len[4];
};

__global__ void __launch_bounds__(256) lora_prep_kernel(const __grid_constant__ PrepParams p) {
  __shared__ uint16_t tile[QLORA_MAX_RANK_DEV][34];
  const int KL = 2 * p.rp;
  const int KV = KL / 8;  // 16-byte vectors per packed row
  if (blockIdx.y == 0) {
    // L2x rows n0 .. n0 + 31: transpose of L2[:, n0 .. n0 + 31] through shared memory
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
    if (n0 >= p.o || p.L2x == nullptr) return;
    for (int i = threadIdx.x; i < p.r * 4; i += blockDim.x) {
      const int j = i >> 2, q = i & 3;  // row j of L2, 8 columns n0 + 8q .. n0 + 8q + 7
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n0 + 8 * q < p.o) v = *reinterpret_cast<const uint4*>(p.L2 + static_cast<int64_t>(j) * p.o + n0 + 8 * q);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        tile[j][8 * q + 2 * t] = static_cast<uint16_t>(w[t] & 0xFFFFu);
        tile[j][8 * q + 2 * t + 1] = static_cast<uint16_t>(w[t] >> 16);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * KV; i += blockDim.x) {
      const int dn = i / KV, v = i - dn * KV;
      if (n0 + dn >= p.o) continue;
      const int c = 8 * v;
      const int cc = c < p.rp ? c : c - p.rp;
      uint32_t w[4] = {0, 0, 0, 0};
      if (cc < p.r) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[t] = static_cast<uint32_t>(tile[cc + 2 * t][dn]) | (static_cast<uint32_t>(tile[cc + 2 * t + 1][dn]) << 16);
      }
      *reinterpret_cast<uint4*>(p.L2x + (n0 + dn) * KL + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else if (blockIdx.y == 1) {
    // L1x rows n0 .. n0 + 31: [L1 | 0 | L1 | 0], 16-byte vectors
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
    if (n0 >= p.h || p.L1x == nullptr) return;
    for (int i = threadIdx.x; i < 32 * KV; i += blockDim.x) {
      const int dn = i / KV, v = i - dn * KV;
      if (n0 + dn >= p.h) continue;
      const int c = 8 * v;
      const int cc = c < p.rp ? c : c - p.rp;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (cc < p.r) val = *reinterpret_cast<const uint4*>(p.L1 + (n0 + dn) * p.r + cc);
      *reinterpret_cast<uint4*>(p.L1x + (n0 + dn) * KL + c) = val;
    }
  } else {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float4* z = reinterpret_cast<float4*>(p.zero_ptr[b]);
      if (z == nullptr) continue;
      const int64_t n4 = p.zero_len[b] / 4;
      for (int64_t i = tid; i < n4; i += stride) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

}  // namespace qlora

namespace qlora {

// ====================================================================== small-M forward

// D^T[n][m] = sum_k W'[k][n] X[m][k] (+ LoRA extension) for M <= 32 tokens:
// the dequantized weight is the 128-row tcgen05 A operand, the tokens are N.
//
// The weight tile never passes through shared memory in bf16: expander
// threads write it straight into tensor memory, from where tcgen05.mma reads
// its A operand.  Shared-memory bandwidth is left to the code lookups (the
// 64 KB pair table, one conflict-free 8-byte load per two weights), the TMA
// fills and the tokens read as the B operand.
//
// Persistent stream-K schedule: the (128-row tile, 64-wide K unit) units of
// the whole problem, LoRA units included, are split evenly over one CTA per
// SM, so every SM streams the same number of weight bytes.  A CTA's units form
// one or more segments (runs within one tile); each segment accumulates in one
// of two TMEM buffers and is added to Y (fp32, zeroed beforehand) with red.add
// by 4 epilogue warps while the next segment proceeds.
//
// Roles (768 threads): warp 0 lane 0 streams codes + X (or, for LoRA units,
// s T hi/lo + the L2 tile) through a SK_CSTAGES-deep TMA ring; warp 1 lane 0
// issues tcgen05.mma; warps 4..19 form four expander groups of four warps
// (one warp per TMEM lane quarter, one thread per weight row), group g taking
// the main (weight) units g, g + 4, ... of the CTA and computing each row's
// block constant c' itself; warps 20..23 drain TMEM.  Unit n uses ring slot
// n mod SK_CSTAGES for its codes, its tokens and its TMEM A columns.  The MMA
// warp commits once per batch of SK_BATCH units (a commit stalls the issuing
// thread) to one of SK_NDONE batch barriers; a slot is free again once the
// batch of its previous unit is done.
//
// Shared memory: [start, T) holds the LoRA A ring and the barriers, where T
// is the first 64 KB-aligned window address at or after them; [T, T + 64 KB)
// the pair table; the code/X ring follows it.
constexpr int SK_BN = 128;                          // weight rows per tile (MMA M)
constexpr int SK_BK = 64;                           // K per unit: one 64-block per row
constexpr int SK_CSTAGES = 12;                      // ring depth: code/X slots = TMEM A slots
constexpr int SK_BATCH = 6;                         // units per MMA commit
constexpr int SK_NDONE = SK_CSTAGES / SK_BATCH;     // batch-done barriers
constexpr int SK_ESTAGES = 2;                       // LoRA A ring depth
constexpr int SK_GROUPS = 4;                        // expander groups
constexpr int SK_EPI_WARP0 = 4 + 4 * SK_GROUPS;     // first of the 4 epilogue warps
constexpr int SK_THREADS = 32 * (SK_EPI_WARP0 + 4);
constexpr int SK_X_BYTES = 32 * SK_BK * 2;          // up to 32 tokens x 64 K: 4 KB
constexpr int SK_CODE_BYTES = SK_BN * SK_BK / 2;    // 128 rows x 32 bytes: 4 KB
constexpr int SK_CSLOT = SK_X_BYTES + SK_CODE_BYTES;
constexpr int SK_EA_BYTES = SK_BN * SK_BK * 2;      // LoRA A tile (L2 rows): 16 KB
constexpr int SK_BAR_BYTES = 1024;
constexpr int SK_LOW_BYTES = SK_ESTAGES * SK_EA_BYTES + SK_BAR_BYTES;
// The whole window a launch may need (the table at 64 KB, the ring after it).
constexpr int SK_SMEM_BYTES = 2 * static_cast<int>(kPairTabBytes) + SK_CSTAGES * SK_CSLOT;
constexpr uint32_t SK_TMEM_COLS = 512;
constexpr uint32_t SK_TMEM_A0 = 64;                 // columns [0, 64): the two accumulators
static_assert(SK_TMEM_A0 + SK_CSTAGES * (SK_BK / 2) <= SK_TMEM_COLS, "TMEM ring");
static_assert(SK_CSTAGES % SK_BATCH == 0, "batches tile the ring");
static_assert(SK_ESTAGES * SK_EA_BYTES + SK_BAR_BYTES + 1024 <= 65536 - 4096, "ring below the table");

struct SmallMParams {
  int M;               // tokens
  int N;               // output features o
  int nmma;            // MMA N: tokens rounded up to 16 (16 or 32)
  int k_units;         // main units per tile: h / 64
  int ext_units;       // LoRA extension units per tile
  int blocks_per_row;  // h / 64
  int64_t units;       // tiles * (k_units + ext_units)
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  const float* absmax32;  // single-level constants (no double quantization), or null
  float* out;          // fp32 [M][N], accumulated
  float codebook[16];
};

// Walks the (tile, k-unit) units of a contiguous range without divisions.
struct UnitCursor {
  int tile, k, S_t;
  __device__ __forceinline__ void init(int64_t u0, int units_per_tile) {
    S_t = units_per_tile;
    tile = static_cast<int>(u0 / units_per_tile);
    k = static_cast<int>(u0 - static_cast<int64_t>(tile) * units_per_tile);
  }
  __device__ __forceinline__ void next() {
    if (++k == S_t) {
      k = 0;
      ++tile;
    }
  }
};

// Ring position (slot, phase parity) of a sequence index, advanced without
// divisions.
template <int S>
struct RingPos {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int step) {
    slot += step;
    while (slot >= S) {
      slot -= S;
      phase ^= 1u;
    }
  }
};

// Walks the main (weight) units of a CTA's range that belong to one expander
// group, SK_GROUPS main units at a time: unit index n (position in the
// range), main-unit index m, tile, k, and the code/X ring position of n.
template <int S>
struct GroupCursorT {
  int tile, k, n, m, n_units, k_units, ext_units;
  RingPos<S> cr;
  // Main units are consecutive except for the ext_units LoRA units that
  // follow the last K unit of every tile.
  __device__ __forceinline__ void step(int d) {
    k += d;
    n += d;
    m += d;
    int extra = 0;
    while (k >= k_units) {
      k -= k_units;
      ++tile;
      extra += ext_units;
    }
    n += extra;
    cr.advance(d + extra);
  }
  __device__ __forceinline__ void init(int64_t u0, int n_units_, int k_units_, int ext_units_, int group) {
    const int S_t = k_units_ + ext_units_;
    n_units = n_units_;
    k_units = k_units_;
    ext_units = ext_units_;
    tile = static_cast<int>(u0 / S_t);
    k = static_cast<int>(u0 - static_cast<int64_t>(tile) * S_t);
    n = 0;
    m = 0;
    if (k >= k_units) {  // the range starts on LoRA units: skip to the next tile
      n = S_t - k;
      cr.advance(n);
      k = 0;
      ++tile;
    }
    step(group);
  }
  __device__ __forceinline__ bool valid() const { return n < n_units; }
};
using GroupCursor = GroupCursorT<SK_CSTAGES>;

// Waits until ring slot n % SK_CSTAGES is free for unit n: the batch of its
// previous unit n - SK_CSTAGES is done.  That batch uses the same barrier as
// unit n's batch, one phase earlier (a fresh barrier passes the first wait).
__device__ __forceinline__ bool slot_free_wait(uint64_t* done, int n, int tag) {
  const int b = n / SK_BATCH;
  return mbar_wait(&done[b % SK_NDONE], ((b / SK_NDONE) & 1) ^ 1, tag);
}

__global__ void __launch_bounds__(SK_THREADS, 1)
    small_m_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmL2x, const __grid_constant__ CUtensorMap tmTT,
                       const __grid_constant__ SmallMParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t r0 = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  const uint32_t toff = pair_tab_offset(smem_raw, r0 + SK_LOW_BYTES);
  if (toff + kPairTabBytes + SK_CSTAGES * SK_CSLOT > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusSmemLayout);
    return;
  }
  uint8_t* sE = smem_raw + r0;                               // LoRA A ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + SK_ESTAGES * SK_EA_BYTES);
  uint8_t* tab = smem_raw + toff;                            // pair table
  uint8_t* sC = tab + kPairTabBytes;                         // code + X ring (1024-aligned)
  uint64_t* full = bars;                                     // TMA bytes of a slot
  uint64_t* afull = full + SK_CSTAGES;                       // expanding group's 4 warps (or the producer)
  uint64_t* done = afull + SK_CSTAGES;                       // MMA commit of a batch of units
  uint64_t* eempty = done + SK_NDONE;                        // MMA commit: LoRA A slot reusable
  uint64_t* accf = eempty + SK_ESTAGES;                      // accumulator ready (MMA commit)
  uint64_t* acce = accf + 2;                                 // accumulator drained (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S_t = p.k_units + p.ext_units;
  const int64_t G = gridDim.x;
  const int64_t u0 = p.units * blockIdx.x / G;
  const int64_t u1 = p.units * (blockIdx.x + 1) / G;
  const int n_units = static_cast<int>(u1 - u0);
  const uint32_t x_bytes = static_cast<uint32_t>(p.nmma) * SK_BK * 2;

  fill_pair_table(tab, p.codebook);
  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_CSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
    }
    for (int s = 0; s < SK_NDONE; ++s) mbar_init(&done[s], 1);
    for (int s = 0; s < SK_ESTAGES; ++s) mbar_init(&eempty[s], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&accf[s], 1);
      mbar_init(&acce[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, SK_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && n_units > 0) {
      // ---------------- producer: codes + X, or s T (hi/lo) + the L2 tile
      tma_prefetch_map(&tmX);
      tma_prefetch_map(&tmC);
      int issued = 0, ext = 0;
      UnitCursor cur;
      cur.init(u0, S_t);
      for (int n = 0; n < n_units; ++n, cur.next()) {
        const int cs = n % SK_CSTAGES;
        // units of one batch become free together: check once per batch
        if ((n % SK_BATCH == 0 || n == 0) && !slot_free_wait(done, n, 1)) break;
        uint8_t* slot = sC + cs * SK_CSLOT;
        if (cur.k < p.k_units) {
          mbar_arrive_expect_tx(&full[cs], x_bytes + SK_CODE_BYTES);
          tma_load_2d(slot, &tmX, &full[cs], cur.k * SK_BK, 0);
          tma_load_2d(slot + SK_X_BYTES, &tmC, &full[cs], cur.k * (SK_BK / 2), cur.tile * SK_BN);
        } else {
          const int es = ext % SK_ESTAGES;
          if (!mbar_wait(&eempty[es], ((ext / SK_ESTAGES) & 1) ^ 1, 2)) break;
          const int ke = cur.k - p.k_units;
          mbar_arrive_expect_tx(&full[cs], x_bytes + SK_EA_BYTES);
          tma_load_2d(slot, &tmTT, &full[cs], ke * SK_BK, 0);
          tma_load_2d(sE + es * SK_EA_BYTES, &tmL2x, &full[cs], ke * SK_BK, cur.tile * SK_BN);
          // A LoRA unit has no expander group: stand in for its 4 warps, so
          // that every slot's afull barrier advances one phase per unit.
          mbar_arrive_count(&afull[cs], 4);
          ++ext;
        }
        issued = n + 1;
      }
      // No TMA load may still be landing when the CTA exits: wait for the last
      // phase of every slot used (earlier phases of a slot must not be waited
      // on, their parity repeats).
      for (int n = issued - SK_CSTAGES > 0 ? issued - SK_CSTAGES : 0; n < issued; ++n)
        mbar_wait(&full[n % SK_CSTAGES], (n / SK_CSTAGES) & 1, 3);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_units > 0) {
      // ---------------- MMA issuer: one segment (run of units in one tile)
      // at a time, its weight units in chunks that never cross a commit batch
      // (SK_BATCH units of the ring).  After tcgen05.mma a thread's shared-
      // memory accesses (barrier tests included) come back only after ~0.1 us,
      // so each chunk costs one batched test of all its slots (blocking waits
      // only if a slot is not ready), then the chunk's MMAs back to back with
      // no shared-memory access in between, then one commit.
      const uint32_t idesc = idesc_bf16(128, p.nmma, false, false);
      const uint64_t bdesc0 = sw128_desc(smem_u32(sC), 16, 1024);
      const uint32_t afull0 = smem_u32(afull), full0 = smem_u32(full);
      UnitCursor c0;
      c0.init(u0, S_t);
      int n = 0, k = c0.k, ext = 0;
      RingPos<SK_CSTAGES> rp;
      bool ok = true;
      for (int seg = 0; n < n_units && ok; ++seg, k = 0) {
        const int seg_end = k + (S_t - k < n_units - n ? S_t - k : n_units - n);  // one past the last k
        if (seg >= 2 && !mbar_wait(&acce[seg & 1], ((seg >> 1) - 1) & 1, 5)) break;
        const uint32_t d = tmem + static_cast<uint32_t>(seg & 1) * 32u;
        const int main_end = seg_end < p.k_units ? seg_end : p.k_units;
        uint32_t acc = 0;
        while (k < main_end) {
          int c = SK_BATCH - n % SK_BATCH;  // up to the end of the commit batch
          if (c > main_end - k) c = main_end - k;
          // batched readiness test of the chunk's slots (padded by repeating the last)
          uint32_t bars[12], pars[12];
          {
            RingPos<SK_CSTAGES> w = rp;
#pragma unroll
            for (int i = 0; i < 6; ++i) {
              bars[2 * i] = afull0 + 8u * w.slot;
              bars[2 * i + 1] = full0 + 8u * w.slot;
              pars[2 * i] = pars[2 * i + 1] = w.phase;
              if (i + 1 < c) w.advance(1);
            }
          }
          if (!mbar_test12(bars, pars)) {
            // the expanders waited for the slot's fill before arriving
            RingPos<SK_CSTAGES> w = rp;
            for (int i = 0; i < c && ok; ++i, w.advance(1))
              ok = mbar_wait(&afull[w.slot], w.phase, 7) && mbar_wait(&full[w.slot], w.phase, 6);
            if (!ok) break;
          }
          tc_fence_after();
          for (int i = 0; i < c; ++i, ++k, ++n, rp.advance(1)) {
            const uint32_t a_col = tmem + SK_TMEM_A0 + static_cast<uint32_t>(rp.slot) * (SK_BK / 2);
            const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(rp.slot * (SK_CSLOT >> 4));
#pragma unroll
            for (int kk = 0; kk < SK_BK / 16; ++kk)
              umma_bf16_tmem_a(d, a_col + kk * 8, bdesc + 2 * kk, idesc, acc | kk);
            acc = 1;
          }
          if ((n - 1) % SK_BATCH == SK_BATCH - 1 || n == n_units) umma_commit(&done[((n - 1) / SK_BATCH) % SK_NDONE]);
        }
        if (!ok) break;
        // the segment's LoRA units (A = L2 tile, B = s T hi/lo)
        for (; k < seg_end; ++k, ++n, rp.advance(1)) {
          const int cs = rp.slot;
          if (!mbar_wait(&full[cs], rp.phase, 6)) {
            ok = false;
            break;
          }
          const int es = ext % SK_ESTAGES;
          tc_fence_after();
          const uint64_t adesc = sw128_desc(smem_u32(sE + es * SK_EA_BYTES), 16, 1024);
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(cs * (SK_CSLOT >> 4));
#pragma unroll
          for (int kk = 0; kk < SK_BK / 16; ++kk) umma_bf16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, acc | kk);
          acc = 1;
          umma_commit(&eempty[es]);
          ++ext;
          if ((n % SK_BATCH) == SK_BATCH - 1 || n == n_units - 1) umma_commit(&done[(n / SK_BATCH) % SK_NDONE]);
        }
        if (!ok) break;
        umma_commit(&accf[seg & 1]);
      }
    }
  } else if (warp >= 4 && warp < SK_EPI_WARP0) {
    // ---------------- expanders: thread (group, quarter, lane) owns weight row
    // tile * 128 + e of its group's units and writes the row's 64 expanded
    // K values to TMEM lane e (32 columns of the unit's A slot).
    const int grp = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int e = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + SK_TMEM_A0;
    const uint32_t key = pair_key(tab, lane);
    const uint32_t swz = static_cast<uint32_t>((e >> 2) & 1) << 4;  // 32-byte swizzle of the code tile
    const float mu = p.absmax32 ? 0.0f : __ldg(p.dq_mean);
    ConstCache cc;
    // Block constants ride a register ring kPre of the group's units ahead of
    // the expansion (the loop is unrolled by kPre so every ring index is
    // static), so that their global-load latency is covered by several units.
    constexpr int kPre = 2;
    uint32_t e8[kPre];
    float sc[kPre];
    GroupCursor cur, pf;
    cur.init(u0, n_units, p.k_units, p.ext_units, grp);
    pf = cur;
    ConstWindow cw;
    const int64_t nblk = static_cast<int64_t>(p.N) * p.blocks_per_row;
    auto fetch = [&](uint32_t& eo, float& so) {
      eo = 0;
      so = 0.0f;
      const int row = pf.tile * SK_BN + e;
      if (pf.valid() && row < p.N) {
        const int64_t blk = static_cast<int64_t>(row) * p.blocks_per_row + pf.k;
        if (p.absmax32)
          so = __ldg(p.absmax32 + blk);  // the block constant itself
        else
          cw.get(p.absmax_fp8, p.dq_scale, nblk, blk, eo, so);
      }
      pf.step(SK_GROUPS);
    };
#pragma unroll
    for (int t = 0; t < kPre; ++t) fetch(e8[t], sc[t]);
    bool ok = true;
    while (ok) {
#pragma unroll
      for (int t = 0; t < kPre; ++t) {
        if (!cur.valid()) {
          ok = false;
          break;
        }
        const int cs = cur.cr.slot;
        const int row = cur.tile * SK_BN + e;
        const uint32_t e_now = e8[t];
        const float s_now = sc[t];
        fetch(e8[t], sc[t]);
        const uint64_t cp2 = dup_f32x2(
            row < p.N ? (p.absmax32 ? s_now : cc.constant(static_cast<uint8_t>(e_now), s_now, mu)) : 0.0f);
        if (!warp_wait(&full[cs], cur.cr.phase, 8)) {
          ok = false;
          break;
        }
        const uint8_t* crow = sC + cs * SK_CSLOT + SK_X_BYTES + e * 32;
        const uint4 w0 = *reinterpret_cast<const uint4*>(crow + swz);
        const uint4 w1 = *reinterpret_cast<const uint4*>(crow + (swz ^ 16u));
        // The full slot implies its previous unit's batch is done (the fill
        // waited for it), so the MMA that read these TMEM columns has finished.
        tc_fence_after();
        const uint32_t ta = t_lane + static_cast<uint32_t>(cs) * (SK_BK / 2);
        uint32_t v[16];
        {
          const uint4 a = word_dequant(w0.x, key, cp2), b = word_dequant(w0.y, key, cp2);
          const uint4 c = word_dequant(w0.z, key, cp2), d = word_dequant(w0.w, key, cp2);
          v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
          v[8] = c.x, v[9] = c.y, v[10] = c.z, v[11] = c.w, v[12] = d.x, v[13] = d.y, v[14] = d.z, v[15] = d.w;
        }
        tmem_st16(ta, v);
        {
          const uint4 a = word_dequant(w1.x, key, cp2), b = word_dequant(w1.y, key, cp2);
          const uint4 c = word_dequant(w1.z, key, cp2), d = word_dequant(w1.w, key, cp2);
          v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
          v[8] = c.x, v[9] = c.y, v[10] = c.z, v[11] = c.w, v[12] = d.x, v[13] = d.y, v[14] = d.z, v[15] = d.w;
        }
        tmem_st16(ta + 16, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[cs]);
        cur.step(SK_GROUPS);
      }
    }
  } else if (warp >= SK_EPI_WARP0) {
    // ---------------- epilogue: add each finished segment into Y
    const int q = warp & 3;
    int seg = -1;
    UnitCursor cur;
    cur.init(u0, S_t);
    for (int n = 0; n < n_units; ++n, cur.next()) {
      if (n == 0 || cur.k == 0) ++seg;
      const bool last = (n == n_units - 1) || (cur.k == S_t - 1);
      if (!last) continue;
      const int buf = seg & 1;
      if (!warp_wait_sleep(&accf[buf], (seg >> 1) & 1, 11)) break;
      tc_fence_after();
      const int col = cur.tile * SK_BN + q * 32 + lane;
      for (int c = 0; c < p.nmma / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 32 + c * 16, r);
        tmem_ld_wait();
        if (col < p.N) {
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int m = c * 16 + t;
            if (m < p.M) atomicAdd(p.out + static_cast<int64_t>(m) * p.N + col, __uint_as_float(r[t]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, SK_TMEM_COLS);
  }
}

// ====================================================================== small-M forward, register-fed tensor cores

// For M <= 16 tokens the forward is a weight stream with a few dot products
// per weight.  Each weight is dequantized to W' = bf16(q[code] * c') (the
// doubleDequant of the key-formula section, rounded to bf16 per element, the
// compute type of its data-type table) straight into the A-fragment registers
// of mma.sync.m16n8k16 (bf16 x bf16, fp32 accumulation), whose N = 8 columns
// are the tokens (two MMAs per fragment for 9 .. 16 tokens).  The fragments
// never pass through shared or tensor memory and every warp issues its own
// MMAs: per weight the only shared-memory traffic is the pair-table lookup
// (one conflict-free 8-byte load per code byte) and the code tile itself.
//
// K order inside a 64-block.  Fragment lane t (= lane % 4) supplies the K
// slots {2t, 2t+1, 2t+8, 2t+9} of an m16n8k16 step; here lane t takes the
// block's code bytes 8t .. 8t+7 (16 consecutive weights of each of its two
// rows), byte 2s + p feeding step s, slot pair p.  A dot product does not
// depend on the order of its terms and the token fragment follows the same
// map, so a lane reads one 8-byte code word per row and 32 consecutive bytes
// of its token's row per block.
//
// Stream-K over (128-row tile, 256-wide K unit) units, split evenly over one
// CTA per SM.  Roles (768 threads): lanes 0 .. SD_PRODUCERS-1 of warp 0 stream
// each unit's code tile (TMA, 128 x 128-byte box, 128-byte swizzle) and its
// token slice (TMA of X, box {64 K, 4 blocks, M tokens}, 128-byte swizzle)
// into a ring of up to SD_MAX_STAGES slots that fill the shared memory below
// and above the 64 KB-aligned pair table; warps 1 .. 16 form SD_GROUPS groups
// of four warps taking the units round-robin, warp w of a group owning rows
// 32 w .. 32 w + 31 of the unit (two 16-row fragments, fragment rows g and
// g + 8 being rows 2g and 2g + 1 of their half).  Lane (g, t) computes
// the four block constants c' of one of those 32 rows and hands them to the
// lanes that need them by shuffles.  Partial sums go to Y with red.add when
// the group's next unit starts another tile.  Warps 17 .. 19 sum the partials
// of T = X L1 (a fixed order, the same in every CTA) and add s T L2 for an
// even share of the output rows, from fp32 T and the bf16 L2 as given.
constexpr int SD_UNIT_K = 256;                          // K per unit: 128-byte code rows
constexpr int SD_UNIT_BLOCKS = SD_UNIT_K / 64;
constexpr int SD_CODE_BYTES = SK_BN * SD_UNIT_K / 2;    // 16 KB, 128-byte swizzle
constexpr int SD_X_ROW_BYTES = 64 * 2;                  // one token's slice of one block
constexpr int SD_MAX_STAGES = 8;
constexpr int SD_PRODUCERS = 2;                         // issuing lanes of the producer warp
constexpr int SD_SMEM_BYTES = 227 * 1024;               // all of it: slots sit below and above the table
constexpr int SD_BAR_BYTES = 1024;                      // barriers; T follows them
constexpr int SD_GROUPS = 4;                            // groups of 4 MMA warps: warps 1 .. 16
constexpr int SD_LORA_WARP0 = 1 + 4 * SD_GROUPS;        // warps 17 .. 19: the LoRA term
constexpr int SD_THREADS = 640;
constexpr int SD_LORA_THREADS = SD_THREADS - 32 * SD_LORA_WARP0;
constexpr int SD_MAX_TOKENS = 16;
static_assert(SD_LORA_THREADS >= 32, "at least one LoRA warp");
static_assert(SD_MAX_STAGES % SD_PRODUCERS == 0, "each producer lane owns fixed slots");

struct DecodeParams {
  int M;               // tokens, 1 .. SD_MAX_TOKENS
  int N;               // output features o
  int k_units;         // ceil(h / SD_UNIT_K)
  int blocks_per_row;  // h / 64
  int r;               // LoRA rank
  float s;             // LoRA scale
  int64_t units;       // tiles * k_units
  int slot_bytes;      // code tile + token slice (M x 512 B), a multiple of 1 KB
  int low_bytes;       // barriers + a copy of T (M r fp32), a multiple of 1 KB
  const float* P;      // partials of X L1, fp32 [n_part][M][r], summed in order
  int n_part;
  float* T_out;        // X L1, fp32 [M][r], written by CTA 0 (optional)
  const uint16_t* L2;  // bf16 [r][o]
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  const float* absmax32;  // single-level constants (no double quantization), or null
  float* out;          // fp32 [M][N], zeroed beforehand, accumulated
  float codebook[16];
};

// D (16 x 8, fp32) += A (16 x 16, bf16, row) * B (16 x 8, bf16, col).
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Ring position with a ring size known only at run time.
struct RingPosDyn {
  int slot = 0;
  uint32_t phase = 0;
  int S = 1;
  __device__ __forceinline__ void advance(int step) {
    slot += step;
    while (slot >= S) {
      slot -= S;
      phase ^= 1u;
    }
  }
};

// The units of a CTA's range that belong to one group: every SD_GROUPS-th,
// with the (tile, k) position and the ring position of each.
struct DecodeCursor {
  int tile, k, n, n_units, k_units;
  RingPosDyn cr;
  __device__ __forceinline__ void step(int d) {
    k += d;
    n += d;
    while (k >= k_units) {
      k -= k_units;
      ++tile;
    }
    cr.advance(d);
  }
  __device__ __forceinline__ void init(int64_t u0, int n_units_, int k_units_, int group, int S) {
    n_units = n_units_;
    k_units = k_units_;
    tile = static_cast<int>(u0 / k_units_);
    k = static_cast<int>(u0 - static_cast<int64_t>(tile) * k_units_);
    n = 0;
    cr.S = S;
    step(group);
  }
  __device__ __forceinline__ bool valid() const { return n < n_units; }
};

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// NG token groups of 8 (NG = 1: M <= 8, NG = 2: M <= 16).
template <int NG>
__global__ void __launch_bounds__(SD_THREADS, 1)
    small_m_mma_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t r0 = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  const uint32_t lo0 = r0 + static_cast<uint32_t>(p.low_bytes);
  const uint32_t toff = pair_tab_offset(smem_raw, lo0);
  const uint32_t sb = static_cast<uint32_t>(p.slot_bytes);
  const int n_lo = static_cast<int>((toff - lo0) / sb);
  const uint32_t hi0 = toff + kPairTabBytes;
  const uint32_t dyn = dynamic_smem_bytes();
  const int n_hi = hi0 < dyn ? static_cast<int>((dyn - hi0) / sb) : 0;
  int S = n_lo + n_hi;
  S = S < SD_MAX_STAGES ? S : SD_MAX_STAGES;
  S -= S % SD_PRODUCERS;
  if (S < SD_PRODUCERS || toff + kPairTabBytes > dyn) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusSmemLayout);
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + r0);  // TMA bytes of a slot
  uint64_t* empty = full + SD_MAX_STAGES;                         // the group's 4 warps
  uint8_t* tab = smem_raw + toff;
  // byte offset from smem_raw of ring slot s (1 KB aligned, as the 128-byte swizzle needs)
  auto slot_off = [&](int s) -> uint32_t {
    return s < n_lo ? lo0 + static_cast<uint32_t>(s) * sb : hi0 + static_cast<uint32_t>(s - n_lo) * sb;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t u0 = p.units * blockIdx.x / G;
  const int64_t u1 = p.units * (blockIdx.x + 1) / G;
  const int n_units = static_cast<int>(u1 - u0);

  fill_pair_table(tab, p.codebook);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // Launched as a dependent of rank_r_small_kernel, which zeroes the output and
  // writes the partials of T: only the threads that touch those wait for it
  // (griddepcontrol.wait, before the first flush and before the partials are
  // read); the weight and token stream does not depend on it and starts now.

  if (warp == 0) {
    if (lane < SD_PRODUCERS && lane < n_units) {
      // ---------------- producers: lane j issues units j, j + SD_PRODUCERS, ...
      if (lane == 0) {
        tma_prefetch_map(&tmC);
        tma_prefetch_map(&tmX);
      }
      const uint32_t tx = static_cast<uint32_t>(SD_CODE_BYTES + p.M * SD_UNIT_BLOCKS * SD_X_ROW_BYTES);
      int issued = -1;
      UnitCursor cur;
      cur.init(u0 + lane, p.k_units);
      RingPosDyn rp;
      rp.S = S;
      rp.advance(lane);
      for (int n = lane; n < n_units; n += SD_PRODUCERS) {
        if (!mbar_wait(&empty[rp.slot], rp.phase ^ 1u, 1)) break;
        uint8_t* slot = smem_raw + slot_off(rp.slot);
        mbar_arrive_expect_tx(&full[rp.slot], tx);
        tma_load_2d(slot, &tmC, &full[rp.slot], cur.k * (SD_UNIT_K / 2), cur.tile * SK_BN);
        tma_load_3d(slot + SD_CODE_BYTES, &tmX, &full[rp.slot], 0, cur.k * SD_UNIT_BLOCKS, 0);
        issued = n;
        for (int i = 0; i < SD_PRODUCERS; ++i) cur.next();
        rp.advance(SD_PRODUCERS);
      }
      // No copy of this lane may still be landing when the CTA exits: wait for
      // the last phase of each of its slots that was used (S is a multiple of
      // SD_PRODUCERS, so slot n % S belongs to lane n % SD_PRODUCERS alone).
      int first = issued - S + SD_PRODUCERS;
      if (first < lane) first = lane;
      for (int n = first; n <= issued; n += SD_PRODUCERS) mbar_wait(&full[n % S], (n / S) & 1, 3);
    }
  } else if (warp < SD_LORA_WARP0) {
    // ---------------- MMA warps: warp wq of group grp owns rows 32 wq .. 32 wq + 31
    // of its units; fragment rows g and g + 8 of each 16-row half rt
    const int grp = (warp - 1) >> 2;
    const int wq = (warp - 1) & 3;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t key = pair_key(tab, lane);
    const float mu = p.absmax32 ? 0.0f : __ldg(p.dq_mean);
    const uint32_t smem_base = smem_u32(smem_raw);
    ConstCache cc;
    // the row (within the 128-row tile) whose block constants this lane computes:
    // half rt = t >> 1, row 2g + (t & 1) of the half (fragment row g or g + 8)
    const int own_row = 32 * wq + 16 * (t >> 1) + 2 * g + (t & 1);
    constexpr int kPre = 2;
    // The unit's 4 block constants of own_row, loaded kPre units ahead and
    // decoded when the unit is expanded.  Double-quantized: w[0] holds the FP8
    // codes of blocks 0 .. 3 (bytes 0 .. 3), w[1] / w[2] the second-level
    // scales of blocks 0 and 3, w[3] the number of leading blocks that share
    // block 0's group.  Single-level: w[b] is block b's fp32 constant.
    struct UnitConst {
      uint32_t w[4];
    };
    UnitConst uc[kPre];
    DecodeCursor cur, pf;
    cur.init(u0, n_units, p.k_units, grp, S);
    pf = cur;
    const bool dq_off = p.absmax32 != nullptr;
    const bool c_vec = (p.blocks_per_row & 3) == 0 &&
                       (dq_off ? (reinterpret_cast<uintptr_t>(p.absmax32) & 15u) == 0
                               : (reinterpret_cast<uintptr_t>(p.absmax_fp8) & 3u) == 0);
    auto fetch = [&](UnitConst& u) {
      const int row = pf.tile * SK_BN + own_row;
      u.w[0] = u.w[1] = u.w[2] = 0u;
      u.w[3] = dq_off ? 0u : static_cast<uint32_t>(SD_UNIT_BLOCKS);
      if (pf.valid() && row < p.N) {
        const int kb0 = pf.k * SD_UNIT_BLOCKS;
        const int nbv = min(SD_UNIT_BLOCKS, p.blocks_per_row - kb0);
        const int64_t b0 = static_cast<int64_t>(row) * p.blocks_per_row + kb0;
        if (dq_off) {
          if (c_vec) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.absmax32) + (b0 >> 2));
            u.w[0] = v.x, u.w[1] = v.y, u.w[2] = v.z, u.w[3] = v.w;
          } else {
#pragma unroll
            for (int b = 0; b < SD_UNIT_BLOCKS; ++b)
              if (b < nbv) u.w[b] = __float_as_uint(__ldg(p.absmax32 + b0 + b));
          }
        } else {
          if (c_vec) {
            u.w[0] = __ldg(reinterpret_cast<const uint32_t*>(p.absmax_fp8) + (b0 >> 2));
          } else {
#pragma unroll
            for (int b = 0; b < SD_UNIT_BLOCKS; ++b)
              if (b < nbv) u.w[0] |= static_cast<uint32_t>(__ldg(p.absmax_fp8 + b0 + b)) << (8 * b);
          }
          u.w[1] = __float_as_uint(__ldg(p.dq_scale + (b0 >> 8)));
          u.w[2] = __float_as_uint(__ldg(p.dq_scale + ((b0 + nbv - 1) >> 8)));
          u.w[3] = static_cast<uint32_t>(256 - static_cast<int>(b0 & 255));
        }
      }
      pf.step(SD_GROUPS);
    };
#pragma unroll
    for (int i = 0; i < kPre; ++i) fetch(uc[i]);
    float acc[2][NG][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
      for (int q = 0; q < NG; ++q)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[rt][q][v] = 0.0f;
    int acc_tile = cur.tile;
    auto flush = [&]() {
      pdl_wait();  // the output was zeroed by the rank-r kernel
#pragma unroll
      for (int rt = 0; rt < 2; ++rt) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = acc_tile * SK_BN + 32 * wq + 16 * rt + 2 * g + hh;
#pragma unroll
          for (int q = 0; q < NG; ++q) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int m = 8 * q + 2 * t + c;
              if (n < p.N && m < p.M) atomicAdd(p.out + static_cast<int64_t>(m) * p.N + n, acc[rt][q][2 * hh + c]);
              acc[rt][q][2 * hh + c] = 0.0f;
            }
          }
        }
      }
    };
    bool ok = true;
    while (ok) {
#pragma unroll
      for (int it = 0; it < kPre; ++it) {
        if (!cur.valid()) {
          ok = false;
          break;
        }
        if (cur.tile != acc_tile) {
          flush();
          acc_tile = cur.tile;
        }
        const int cs = cur.cr.slot;
        const UnitConst un = uc[it];
        const int nb = min(SD_UNIT_BLOCKS, p.blocks_per_row - cur.k * SD_UNIT_BLOCKS);
        const bool row_ok = cur.tile * SK_BN + own_row < p.N;
        fetch(uc[it]);
        if (!warp_wait(&full[cs], cur.cr.phase, 8)) {
          ok = false;
          break;
        }
        float cown[SD_UNIT_BLOCKS];
#pragma unroll
        for (int b = 0; b < SD_UNIT_BLOCKS; ++b) {
          float c = 0.0f;
          if (row_ok && b < nb)
            c = dq_off ? __uint_as_float(un.w[b])
                       : cc.constant(static_cast<uint8_t>(un.w[0] >> (8 * b)),
                                     __uint_as_float(b < static_cast<int>(un.w[3]) ? un.w[1] : un.w[2]), mu);
          cown[b] = c;
        }
        const uint32_t slot = smem_base + slot_off(cs);
        const uint32_t xs = slot + SD_CODE_BYTES;
#pragma unroll
        for (int j = 0; j < SD_UNIT_BLOCKS; ++j) {
          if (j >= nb) break;
          // token fragment of block j: token 8 q + g, bf16 pairs 8t .. 8t+7 of the
          // block (16-byte chunks 2t and 2t + 1 of the token's 128-byte row)
          uint32_t xb[NG][8];
#pragma unroll
          for (int q = 0; q < NG; ++q) {
            const int m = 8 * q + g;
            if (m < p.M) {
              const int R = SD_UNIT_BLOCKS * m + j;  // row of the [M][4][64] box
              const uint32_t rb = xs + static_cast<uint32_t>(R) * SD_X_ROW_BYTES;
              const uint32_t sw = static_cast<uint32_t>(R & 7);
              const uint4 v0 = lds_u4(rb + (((2u * t) ^ sw) << 4));
              const uint4 v1 = lds_u4(rb + (((2u * t + 1u) ^ sw) << 4));
              xb[q][0] = v0.x, xb[q][1] = v0.y, xb[q][2] = v0.z, xb[q][3] = v0.w;
              xb[q][4] = v1.x, xb[q][5] = v1.y, xb[q][6] = v1.z, xb[q][7] = v1.w;
            } else {
#pragma unroll
              for (int v = 0; v < 8; ++v) xb[q][v] = 0u;
            }
          }
          // Code bytes 8t .. 8t+7 of block j for the four rows of this lane:
          // fragment row g of half rt is tile row 32 wq + 16 rt + 2g, fragment
          // row g + 8 is the row after it.  Chunk 2j + t/2 of row e sits at
          // position (2j + t/2) ^ (e % 8) (128-byte swizzle); with rows 2g and
          // 2g + 1 the 16 lanes of a half-warp read 16 different bank groups.
          uint2 w[2][2];
          uint64_t cc[2][2];
#pragma unroll
          for (int rt = 0; rt < 2; ++rt) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int e = 32 * wq + 16 * rt + 2 * g + hh;
              const uint32_t coff =
                  ((static_cast<uint32_t>(2 * j + (t >> 1)) ^ static_cast<uint32_t>(e & 7)) << 4) +
                  (static_cast<uint32_t>(t & 1) << 3);
              w[rt][hh] = lds_u2(slot + static_cast<uint32_t>(e) * 128u + coff);
              cc[rt][hh] = dup_f32x2(__shfl_sync(0xFFFFFFFFu, cown[j], g * 4 + 2 * rt + hh));
            }
          }
          // step s takes bytes 2s (slots 2t, 2t+1) and 2s + 1 (slots 2t+8, 2t+9);
          // the two halves' MMAs alternate (independent accumulators)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
              const uint32_t r0w = s < 2 ? w[rt][0].x : w[rt][0].y;
              const uint32_t r1w = s < 2 ? w[rt][1].x : w[rt][1].y;
              uint32_t a0, a1, a2, a3;
              if ((s & 1) == 0) {
                a0 = pair_dequant<0>(r0w, key, cc[rt][0]), a1 = pair_dequant<0>(r1w, key, cc[rt][1]);
                a2 = pair_dequant<1>(r0w, key, cc[rt][0]), a3 = pair_dequant<1>(r1w, key, cc[rt][1]);
              } else {
                a0 = pair_dequant<2>(r0w, key, cc[rt][0]), a1 = pair_dequant<2>(r1w, key, cc[rt][1]);
                a2 = pair_dequant<3>(r0w, key, cc[rt][0]), a3 = pair_dequant<3>(r1w, key, cc[rt][1]);
              }
#pragma unroll
              for (int q = 0; q < NG; ++q)
                mma_16816_bf16(acc[rt][q], a0, a1, a2, a3, xb[q][2 * s], xb[q][2 * s + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[cs]);
        cur.step(SD_GROUPS);
      }
    }
    flush();
  } else {
    // ---------------- LoRA term: T = X L1 from its per-CTA partials (the same
    // fixed order in every CTA), then Y[m][n] += s sum_j T[m][j] L2[j][n] for
    // an even share of the output rows.  The partials are read four columns at
    // a time with eight partials in flight per thread, so the sum costs a few
    // memory latencies whatever M.
    const int tid = threadIdx.x - 32 * SD_LORA_WARP0;
    pdl_wait();  // the partials of T and the zeroed output come from the rank-r kernel
    float* Ts = reinterpret_cast<float*>(smem_raw + r0 + SD_BAR_BYTES);
    const int nt = p.M * p.r;  // a multiple of 8
    const float4* P4 = reinterpret_cast<const float4*>(p.P);
    for (int q = tid; q < nt / 4; q += SD_LORA_THREADS) {
      float4 a[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      int b = 0;
      for (; b + 8 <= p.n_part; b += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v = __ldg(P4 + static_cast<int64_t>(b + u) * (nt / 4) + q);
          a[u].x += v.x, a[u].y += v.y, a[u].z += v.z, a[u].w += v.w;
        }
      }
      for (; b < p.n_part; ++b) {
        const float4 v = __ldg(P4 + static_cast<int64_t>(b) * (nt / 4) + q);
        a[0].x += v.x, a[0].y += v.y, a[0].z += v.z, a[0].w += v.w;
      }
#pragma unroll
      for (int u = 4; u > 0; u >>= 1)
#pragma unroll
        for (int i = 0; i < u; ++i)
          a[i].x += a[i + u].x, a[i].y += a[i + u].y, a[i].z += a[i + u].z, a[i].w += a[i + u].w;
      reinterpret_cast<float4*>(Ts)[q] = a[0];
      if (blockIdx.x == 0 && p.T_out != nullptr) reinterpret_cast<float4*>(p.T_out)[q] = a[0];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(SD_LORA_THREADS) : "memory");  // the LoRA warps only
    const int64_t n0 = static_cast<int64_t>(p.N) * blockIdx.x / G;
    const int64_t n1 = static_cast<int64_t>(p.N) * (blockIdx.x + 1) / G;
    constexpr int MT = 8 * NG;
    for (int64_t n = n0 + tid; n < n1; n += SD_LORA_THREADS) {
      float sum[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) sum[m] = 0.0f;
      for (int j = 0; j < p.r; ++j) {
        const float l2 = __uint_as_float(static_cast<uint32_t>(__ldg(p.L2 + static_cast<int64_t>(j) * p.N + n)) << 16);
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < p.M) sum[m] = fmaf(Ts[m * p.r + j], l2, sum[m]);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < p.M) atomicAdd(p.out + static_cast<int64_t>(m) * p.N + n, p.s * sum[m]);
    }
  }
}

// fp32 -> bf16 (round to nearest even), element-wise.
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ in, int64_t n,
                                                          uint16_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
}

// Dropout of the adapter input: Xm = X with the dropped elements set to zero
// (exact in bf16; the 1 / (1 - p) scale is applied to the products instead).
// Eight elements (two Philox draws) per thread and step.
__global__ void __launch_bounds__(256) dropout_mask_kernel(const uint4* __restrict__ X, int64_t nvec,
                                                           uint4* __restrict__ Xm, uint32_t thr, uint64_t seed) {
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 x = __ldg(X + v);
    const uint32_t k0 = dropout_keep4(2 * static_cast<uint64_t>(v), seed, thr);
    const uint32_t k1 = dropout_keep4(2 * static_cast<uint64_t>(v) + 1, seed, thr);
    Xm[v] = make_uint4(keep_pair(x.x, k0), keep_pair(x.y, k0 >> 2), keep_pair(x.z, k1), keep_pair(x.w, k1 >> 2));
  }
}

// T = X L1 for a few tokens (M <= 32), split over K.  A CTA takes
// rank_r_rows(r) consecutive rows of L1: each thread loads its kRankRpt
// 16-byte vectors of them (vector v of rows rl, rl + nrl, ...) up front, so
// one memory latency covers the CTA, and the tokens' slice is staged in
// shared memory.  Per chunk of 4 tokens the thread accumulates 4 x 8 columns
// in fp32 (bf16 x bf16 products are exact) and the row lanes are summed
// through shared memory.  The CTA's sum for (token, column), times `scale`
// (1 / (1 - p) with dropout, whose dropped tokens are zeroed as they are
// staged), is either stored as its partial P[b][m][j] (P given: the consumer
// adds the partials in a fixed order) or added into T (zeroed beforehand)
// with a red.add.
// Also, when given, the grid zeroes zero[0 .. zero_len) (a multiple of 4
// floats): the fp32 accumulator of the decode kernel that follows.
constexpr int kRankRpt = 8;
__host__ __device__ constexpr int rank_r_lanes(int r) { return 256 / (r / 8) < 32 ? 256 / (r / 8) : 32; }
__host__ __device__ constexpr int rank_r_rows(int r) { return rank_r_lanes(r) * kRankRpt; }
__global__ void __launch_bounds__(256) rank_r_small_kernel(const uint16_t* __restrict__ X, int M, int64_t h,
                                                           const uint16_t* __restrict__ L1, int r,
                                                           float* __restrict__ T, float* __restrict__ P,
                                                           float* __restrict__ zero, int64_t zero_len,
                                                           uint32_t mask_thr, uint64_t mask_seed, float scale) {
  __shared__ __align__(16) float red[8192];     // [row lane][4 tokens][r]: nrl * r / 8 <= 256
  __shared__ __align__(16) uint16_t xs[32 * 32 * kRankRpt];  // [M][rows], rows <= 256
  pdl_launch_dependents();  // the decode kernel may start its prologue now
  if (zero != nullptr) {
    float4* z = reinterpret_cast<float4*>(zero);
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < zero_len / 4;
         q += static_cast<int64_t>(gridDim.x) * blockDim.x)
      z[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int nv = r >> 3;
  const int nrl = rank_r_lanes(r);
  const int rows = nrl * kRankRpt;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * rows;
  const int nrow = static_cast<int>(h - i0 < rows ? h - i0 : rows);
  if (nrow <= 0) return;
  const int v = threadIdx.x % nv, rl = threadIdx.x / nv;
  const bool active = rl < nrl && (T != nullptr || P != nullptr);
  const uint4* l1 = reinterpret_cast<const uint4*>(L1 + i0 * r) + v;
  uint4 lv[kRankRpt];
#pragma unroll
  for (int u = 0; u < kRankRpt; ++u) {
    const int i = rl + u * nrl;
    lv[u] = active && i < nrow ? __ldg(l1 + static_cast<int64_t>(i) * nv) : make_uint4(0u, 0u, 0u, 0u);
  }
  // the tokens' slice as 16-byte vectors (rows and h are multiples of 8, so nrow and every
  // vector start are too)
  const int nvec = nrow / 8;
#pragma unroll 4
  for (int q = threadIdx.x; q < M * nvec; q += blockDim.x) {
    const int m = q / nvec, c = q - m * nvec;
    uint4 v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * h + i0) + c);
    if (mask_thr) {  // dropout of the adapter input: elements i .. i + 7 of X
      const uint64_t i = static_cast<uint64_t>(m) * h + i0 + 8 * c;
      const uint32_t k0 = dropout_keep4(i >> 2, mask_seed, mask_thr), k1 = dropout_keep4((i >> 2) + 1, mask_seed, mask_thr);
      v = make_uint4(keep_pair(v.x, k0), keep_pair(v.y, k0 >> 2), keep_pair(v.z, k1), keep_pair(v.w, k1 >> 2));
    }
    *reinterpret_cast<uint4*>(xs + m * rows + 8 * c) = v;
  }
  __syncthreads();
  if (T == nullptr && P == nullptr) return;
  for (int m0 = 0; m0 < M; m0 += 4) {
    if (active) {
      float acc[4][8];
#pragma unroll
      for (int mm = 0; mm < 4; ++mm)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[mm][c] = 0.0f;
#pragma unroll
      for (int u = 0; u < kRankRpt; ++u) {
        const int i = rl + u * nrl;
        const uint32_t lw[4] = {lv[u].x, lv[u].y, lv[u].z, lv[u].w};
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          // rows past the end hold zero vectors; tokens past M are skipped
          const float x = m0 + mm < M && i < nrow
                              ? __uint_as_float(static_cast<uint32_t>(xs[(m0 + mm) * rows + i]) << 16)
                              : 0.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            acc[mm][2 * c] = fmaf(x, __uint_as_float(lw[c] << 16), acc[mm][2 * c]);
            acc[mm][2 * c + 1] = fmaf(x, __uint_as_float(lw[c] & 0xFFFF0000u), acc[mm][2 * c + 1]);
          }
        }
      }
      // 16-byte stores: a quarter warp writes 8 consecutive vectors (no bank conflicts)
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        float4* d = reinterpret_cast<float4*>(red + (rl * 4 + mm) * r + 8 * v);
        d[0] = make_float4(acc[mm][0], acc[mm][1], acc[mm][2], acc[mm][3]);
        d[1] = make_float4(acc[mm][4], acc[mm][5], acc[mm][6], acc[mm][7]);
      }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < 4 * r; q += blockDim.x) {
      const int mm = q / r, j = q - mm * r;
      if (m0 + mm < M) {
        float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        int k = 0;
        for (; k + 4 <= nrl; k += 4) {
#pragma unroll
          for (int t = 0; t < 4; ++t) s4[t] += red[((k + t) * 4 + mm) * r + j];
        }
        for (; k < nrl; ++k) s4[0] += red[(k * 4 + mm) * r + j];
        const float sum = scale * ((s4[0] + s4[1]) + (s4[2] + s4[3]));
        const int o = (m0 + mm) * r + j;
        if (P != nullptr)
          P[static_cast<int64_t>(blockIdx.x) * M * r + o] = sum;
        else
          atomicAdd(T + o, sum);
      }
    }
    __syncthreads();
  }
}

}  // namespace qlora
