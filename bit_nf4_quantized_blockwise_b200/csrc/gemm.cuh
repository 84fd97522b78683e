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
    const float mu = __ldg(p.dq_mean);
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
    // the TMA 128-byte swizzle (16-byte chunk index XOR row % 8).
    const int code_off0 = kBwd ? kr * 128 + (((2 * atom) ^ (kr & 7)) << 4) : e * 32;
    const int code_off1 = kBwd ? kr * 128 + (((2 * atom + 1) ^ (kr & 7)) << 4) : e * 32 + 16;
    uint32_t boff[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (kBwd) {
        boff[c] = atom * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128 + ((c ^ (kr & 7)) << 4);
      } else {
        boff[c] = (e >> 3) * 1024 + (e & 7) * 128 + ((c ^ (e & 7)) << 4);
      }
    }
    // block constants, prefetched two stages ahead
    uint32_t ec[3] = {0, 0, 0};
    float sc[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (in_range && t < KM) {
        const int64_t blk = block_index(t);
        ec[t] = __ldg(p.absmax_fp8 + blk);
        sc[t] = __ldg(p.dq_scale + (blk >> 8));
      }
    }
    ConstCache cc;
    for (int i = 0; i < KM; ++i) {
      const int s = i % QG_STAGES;
      const uint32_t ph = (i / QG_STAGES) & 1;
      const int cs = i % QG_CSTAGES;
      const uint32_t cph = (i / QG_CSTAGES) & 1;
      if (in_range && i + 2 < KM) {
        const int64_t blk = block_index(i + 2);
        ec[2] = __ldg(p.absmax_fp8 + blk);
        sc[2] = __ldg(p.dq_scale + (blk >> 8));
      }
      Lut16 L;
      build_lut16(q, in_range ? cc.constant(static_cast<uint8_t>(ec[0]), sc[0], mu) : 0.0f, L);
      if (!mbar_wait(&cfull[cs], cph)) break;
      const uint8_t* cbase = sC + cs * QG_CODE_BYTES;
      const uint4 c0 = *reinterpret_cast<const uint4*>(cbase + code_off0);
      const uint4 c1 = *reinterpret_cast<const uint4*>(cbase + code_off1);
      if (!mbar_wait(&empty[s], ph ^ 1)) break;
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
      ec[0] = ec[1];
      ec[1] = ec[2];
      sc[0] = sc[1];
      sc[1] = sc[2];
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
constexpr int TG_SMEM_LIMIT = 200 * 1024;

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
        if (p.transpose_out) {
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (n + t < p.N) atomicAdd(p.out + static_cast<int64_t>(n + t) * p.ld_out + m, __uint_as_float(r[t]));
        } else {
          float* row = p.out + static_cast<int64_t>(m) * p.ld_out + n;
#pragma unroll
          for (int t = 0; t < 16; t += 4)
            if (n + t < p.N)
              red_add_v4(row + t, __uint_as_float(r[t]), __uint_as_float(r[t + 1]), __uint_as_float(r[t + 2]),
                         __uint_as_float(r[t + 3]));
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

// ====================================================================== small element-wise kernels

// TT[m][c] for the LoRA extension of the fused GEMM, row length 2 * rp:
//   c <  r            : hi = bf16(s * T[m][c])
//   rp <= c < rp + r  : lo = bf16(s * T[m][c - rp] - hi)
//   otherwise         : 0
// s * T is one fp32 rounding; hi + lo carries it to ~2^-17 relative.
__global__ void __launch_bounds__(256) lora_split_kernel(const float* __restrict__ T, int64_t M, int r, int rp,
                                                         float s, uint16_t* __restrict__ TT) {
  const int64_t total = M * 2 * rp;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / (2 * rp);
    const int c = static_cast<int>(i - m * 2 * rp);
    const int cc = c < rp ? c : c - rp;
    uint16_t out = 0;
    if (cc < r) {
      const float v = __fmul_rn(s, T[m * r + cc]);
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      out = c < rp ? __bfloat16_as_ushort(hi)
                   : __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi))));
    }
    TT[i] = out;
  }
}

// B_ext[n][c], row length 2 * rp, K-major rows of the LoRA extension:
//   c < r or rp <= c < rp + r : src(n, c mod rp), else 0, where
//   src(n, k) = L[k][n] (transpose = 1, forward: L = L2 [r][N]) or
//   src(n, k) = L[n][k] (transpose = 0, backward: L = L1 [N][r]).
__global__ void __launch_bounds__(256) lora_ext_kernel(const uint16_t* __restrict__ L, int64_t N, int r, int rp,
                                                       int transpose, uint16_t* __restrict__ B) {
  const int64_t total = N * 2 * rp;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / (2 * rp);
    const int c = static_cast<int>(i - n * 2 * rp);
    const int cc = c < rp ? c : c - rp;
    uint16_t v = 0;
    if (cc < r) v = transpose ? L[static_cast<int64_t>(cc) * N + n] : L[n * r + cc];
    B[i] = v;
  }
}

}  // namespace qlora

namespace qlora {

// ====================================================================== small-M forward

// D^T[n][m] = sum_k W'[k][n] X[m][k] (+ LoRA extension) for M <= 64 tokens:
// the dequantized weight is the 128-row tcgen05 A operand, the tokens are N.
// Split-K over the reduction fills the GPU; partial sums go to fp32 with
// red.add.  Codes arrive by TMA through a 6-deep ring; 4 expander warps turn
// one 64-block per thread per stage into the swizzled K-major A tile.
constexpr int SK_BN = 128;
constexpr int SK_BK = 64;
constexpr int SK_STAGES = 6;
constexpr int SK_THREADS = 256;
constexpr int SK_A_BYTES = SK_BN * SK_BK * 2;  // 16 KB
constexpr int SK_B_BYTES = 64 * SK_BK * 2;     // room for up to 64 tokens: 8 KB
constexpr int SK_C_BYTES = SK_BN * SK_BK / 2;  // 4 KB of codes
constexpr int SK_STAGE_BYTES = SK_A_BYTES + SK_B_BYTES + SK_C_BYTES;
constexpr int SK_SMEM_BYTES = SK_STAGES * SK_STAGE_BYTES + 1024 + 256;

struct SmallMParams {
  int M;               // tokens
  int N;               // output features o
  int nmma;            // MMA N: tokens rounded up to 16
  int k_stages;        // h / 64
  int k_per_split;
  int ext_stages;      // LoRA extension stages (split 0 only)
  int blocks_per_row;  // h / 64
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  float* out;          // fp32 [M][N], accumulated
  float codebook[16];
};

__global__ void __launch_bounds__(SK_THREADS, 1)
    small_m_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmL2x, const __grid_constant__ CUtensorMap tmTT,
                       const __grid_constant__ SmallMParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SK_STAGES * SK_STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* aready = bars + SK_STAGES;
  uint64_t* empty = bars + 2 * SK_STAGES;
  uint64_t* accum = bars + 3 * SK_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * SK_STAGES + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * SK_BN;
  const int kz0 = blockIdx.y * p.k_per_split;
  int kz1 = kz0 + p.k_per_split;
  kz1 = kz1 < p.k_stages ? kz1 : p.k_stages;
  const int main_n = kz1 > kz0 ? kz1 - kz0 : 0;
  const int S = main_n + (blockIdx.y == 0 ? p.ext_stages : 0);
  const uint32_t tmem_cols = p.nmma <= 32 ? 32u : 64u;
  const uint32_t x_bytes = static_cast<uint32_t>(p.nmma) * SK_BK * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&aready[s], 4);
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

  if (warp == 0) {
    if (lane == 0 && S > 0) {
      int issued = 0;
      for (int i = 0; i < S; ++i) {
        const int s = i % SK_STAGES;
        const uint32_t ph = (i / SK_STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        uint8_t* st = smem + s * SK_STAGE_BYTES;
        if (i < main_n) {
          const int k = kz0 + i;
          mbar_arrive_expect_tx(&full[s], x_bytes + SK_C_BYTES);
          tma_load_2d(st + SK_A_BYTES, &tmX, &full[s], k * SK_BK, 0);
          tma_load_2d(st + SK_A_BYTES + SK_B_BYTES, &tmC, &full[s], k * (SK_BK / 2), n0);
        } else {
          const int j = i - main_n;
          mbar_arrive_expect_tx(&full[s], SK_A_BYTES + x_bytes);
          tma_load_2d(st, &tmL2x, &full[s], j * SK_BK, n0);
          tma_load_2d(st + SK_A_BYTES, &tmTT, &full[s], j * SK_BK, 0);
        }
        issued = i + 1;
      }
      for (int i = issued - SK_STAGES > 0 ? issued - SK_STAGES : 0; i < issued; ++i)
        mbar_wait(&full[i % SK_STAGES], (i / SK_STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && S > 0) {
      const uint32_t idesc = idesc_bf16(128, p.nmma, false, false);
      for (int i = 0; i < S; ++i) {
        const int s = i % SK_STAGES;
        const uint32_t ph = (i / SK_STAGES) & 1;
        if (!mbar_wait(&full[s], ph)) break;
        if (i < main_n && !mbar_wait(&aready[s], ph)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * SK_STAGE_BYTES);
        const uint32_t b_base = a_base + SK_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < SK_BK / 16; ++kk)
          umma_bf16(tmem, sw128_desc(a_base + kk * 32, 16, 1024), sw128_desc(b_base + kk * 32, 16, 1024), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else if (warp >= 4) {
    const int e = threadIdx.x - 128;  // row n0 + e of W^T
    const bool in_range = n0 + e < p.N;
    const float mu = __ldg(p.dq_mean);
    float q[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = p.codebook[j];
    const int64_t row_blk = static_cast<int64_t>(n0 + e) * p.blocks_per_row;
    uint32_t ecode = 0;
    float scale = 0.0f;
    if (in_range && main_n > 0) {
      ecode = __ldg(p.absmax_fp8 + row_blk + kz0);
      scale = __ldg(p.dq_scale + ((row_blk + kz0) >> 8));
    }
    for (int i = 0; i < main_n; ++i) {
      const int s = i % SK_STAGES;
      const uint32_t ph = (i / SK_STAGES) & 1;
      uint32_t necode = 0;
      float nscale = 0.0f;
      if (in_range && i + 1 < main_n) {
        necode = __ldg(p.absmax_fp8 + row_blk + kz0 + i + 1);
        nscale = __ldg(p.dq_scale + ((row_blk + kz0 + i + 1) >> 8));
      }
      Lut16 L;
      build_lut16(q, in_range ? block_constant(static_cast<uint8_t>(ecode), scale, mu) : 0.0f, L);
      if (!mbar_wait(&full[s], ph)) break;
      uint8_t* st = smem + s * SK_STAGE_BYTES;
      const uint4* csrc = reinterpret_cast<const uint4*>(st + SK_A_BYTES + SK_B_BYTES + e * 32);
      const uint4 c0 = csrc[0], c1 = csrc[1];
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint8_t* arow = st + (e >> 3) * 1024 + (e & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(arow + ((c ^ (e & 7)) << 4)) = lut_lookup8(L, words[c]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[s]);
      ecode = necode;
      scale = nscale;
    }
  }

  if (warp < 4) {
    __syncwarp();
    const bool ok = S > 0 && mbar_wait(accum, 0);
    tc_fence_after();
    if (ok) {
      const int n = n0 + warp * 32 + lane;
      for (int c = 0; c < p.nmma / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 16, r);
        tmem_ld_wait();
        if (n < p.N) {
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int m = c * 16 + t;
            if (m < p.M) atomicAdd(p.out + static_cast<int64_t>(m) * p.N + n, __uint_as_float(r[t]));
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

// fp32 -> bf16 (round to nearest even), element-wise.
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ in, int64_t n,
                                                          uint16_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
}

}  // namespace qlora
