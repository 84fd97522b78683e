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
        e8 = __ldg(p.absmax_fp8 + blk);
        s32 = __ldg(p.dq_scale + (blk >> 8));
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
      build_lut16(q, in_range ? cc.constant(static_cast<uint8_t>(e_now), s_now, mu) : 0.0f, L);
      if (!mbar_wait(&cfull[cs], cph)) {
        ok = false;
        break;
      }
      const uint8_t* cbase = sC + cs * QG_CODE_BYTES;
      const uint4 c0 = *reinterpret_cast<const uint4*>(cbase + code_off0);
      const uint4 c1 = *reinterpret_cast<const uint4*>(cbase + code_off1);
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
//                     32 rows per CTA, transposed through shared memory;
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
    if (n0 >= p.o) return;
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
    if (n0 >= p.h) return;
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
// Persistent stream-K schedule: the (128-row tile, 64-wide K stage) units of
// the whole problem, LoRA stages included, are split evenly over one CTA per
// SM, so every SM streams the same number of weight bytes.  A CTA's units form
// one or more segments (runs within one tile); each segment accumulates in one
// of two TMEM buffers and is added to Y (fp32, zeroed beforehand) with red.add
// by 4 epilogue warps while the next segment proceeds.
//
// Roles (768 threads): warp 0 lane 0 streams codes + X tiles (and the LoRA
// tiles) through an 8-deep TMA ring; warp 2 lane 0 manages the 8-deep A ring (TMA of
// the LoRA weight tiles); warp 1 lane 0 issues tcgen05.mma; warps 4..19
// expand each unit (four threads per 64-block, 16 elements each, so that four
// expander warps per scheduler hide the shared-memory lookup latency); warps
// 20..23 drain TMEM.
constexpr int SK_BN = 128;
constexpr int SK_BK = 64;
constexpr int SK_ASTAGES = 8;
constexpr int SK_CSTAGES = 8;
constexpr int SK_SPLIT = 4;                        // expander threads per weight row
constexpr int SK_EXP_WARPS = 4 * SK_SPLIT;         // 16 expander warps: 4 per scheduler
constexpr int SK_EPI_WARP0 = 4 + SK_EXP_WARPS;     // first of the 4 epilogue warps
constexpr int SK_THREADS = 32 * (SK_EPI_WARP0 + 4);
constexpr int SK_A_BYTES = SK_BN * SK_BK * 2;    // 16 KB dequantized tile
constexpr int SK_X_BYTES = 32 * SK_BK * 2;       // up to 32 tokens: 4 KB
constexpr int SK_CODE_BYTES = SK_BN * SK_BK / 2; // 4 KB of packed codes
constexpr int SK_CSLOT = SK_X_BYTES + SK_CODE_BYTES;
constexpr int SK_SMEM_BYTES = SK_ASTAGES * SK_A_BYTES + SK_CSTAGES * SK_CSLOT + 512 + 1024;

struct SmallMParams {
  int M;               // tokens
  int N;               // output features o
  int nmma;            // MMA N: tokens rounded up to 16 (16 or 32)
  int k_stages;        // main stages per tile: h / 64
  int ext_stages;      // LoRA extension stages per tile
  int blocks_per_row;  // h / 64
  int64_t units;       // tiles * (k_stages + ext_stages)
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  float* out;          // fp32 [M][N], accumulated
  float codebook[16];
};

// 8 codes (one 32-bit word) -> 8 bf16 via the fp32 codebook in shared memory:
// one byte-address op and one LDS per element (at most 16 distinct words per
// warp request, so no bank conflicts), one fp32 multiply, paired rounding.
__device__ __forceinline__ uint4 expand_word_smem(uint32_t qbase, uint32_t w, float cp) {
  uint32_t o[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t a_hi = qbase + (nibble_x4(w, 8 * b + 4));
    const uint32_t a_lo = qbase + (nibble_x4(w, 8 * b));
    float qh, ql;
    asm("ld.shared.f32 %0, [%1];" : "=f"(qh) : "r"(a_hi));
    asm("ld.shared.f32 %0, [%1];" : "=f"(ql) : "r"(a_lo));
    o[b] = pack_bf16x2(__fmul_rn(qh, cp), __fmul_rn(ql, cp));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Walks the (tile, k-stage) units of a contiguous range without divisions.
struct UnitCursor {
  int tile, k, S_t;
  __device__ __forceinline__ void init(int64_t u0, int stages_per_tile) {
    S_t = stages_per_tile;
    tile = static_cast<int>(u0 / stages_per_tile);
    k = static_cast<int>(u0 - static_cast<int64_t>(tile) * stages_per_tile);
  }
  __device__ __forceinline__ void next() {
    if (++k == S_t) {
      k = 0;
      ++tile;
    }
  }
};

__global__ void __launch_bounds__(SK_THREADS, 1)
    small_m_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmL2x, const __grid_constant__ CUtensorMap tmTT,
                       const __grid_constant__ SmallMParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sA = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sC = sA + SK_ASTAGES * SK_A_BYTES;
  float* s_q = reinterpret_cast<float*>(sC + SK_CSTAGES * SK_CSLOT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_q + 16);
  uint64_t* cfull = bars;                         // TMA bytes of a code/X slot
  uint64_t* cempty = cfull + SK_CSTAGES;          // MMA commit + 4 expander warps
  uint64_t* afull = cempty + SK_CSTAGES;          // A producer + 4 expander warps (+ TMA bytes)
  uint64_t* aempty = afull + SK_ASTAGES;          // MMA commit
  uint64_t* accf = aempty + SK_ASTAGES;           // accumulator buffer ready (MMA commit)
  uint64_t* acce = accf + 2;                      // accumulator buffer drained (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S_t = p.k_stages + p.ext_stages;
  const int64_t G = gridDim.x;
  const int64_t u0 = p.units * blockIdx.x / G;
  const int64_t u1 = p.units * (blockIdx.x + 1) / G;
  const int n_units = static_cast<int>(u1 - u0);
  const uint32_t x_bytes = static_cast<uint32_t>(p.nmma) * SK_BK * 2;

  if (threadIdx.x < 16) s_q[threadIdx.x] = p.codebook[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_CSTAGES; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 1 + SK_EXP_WARPS);
    }
    for (int s = 0; s < SK_ASTAGES; ++s) {
      mbar_init(&afull[s], 1 + SK_EXP_WARPS);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&accf[s], 1);
      mbar_init(&acce[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && n_units > 0) {
      // ---------------- codes / X / LoRA-token producer
      int issued = 0;
      UnitCursor cur;
      cur.init(u0, S_t);
      for (int n = 0; n < n_units; ++n, cur.next()) {
        const int tile = cur.tile;
        const int k = cur.k;
        const int cs = n % SK_CSTAGES;
        if (!mbar_wait(&cempty[cs], ((n / SK_CSTAGES) & 1) ^ 1, 1)) break;
        uint8_t* slot = sC + cs * SK_CSLOT;
        if (k < p.k_stages) {
          mbar_arrive_expect_tx(&cfull[cs], x_bytes + SK_CODE_BYTES);
          tma_load_2d(slot, &tmX, &cfull[cs], k * SK_BK, 0);
          tma_load_2d(slot + SK_X_BYTES, &tmC, &cfull[cs], k * (SK_BK / 2), tile * SK_BN);
        } else {
          mbar_arrive_expect_tx(&cfull[cs], x_bytes);
          tma_load_2d(slot, &tmTT, &cfull[cs], (k - p.k_stages) * SK_BK, 0);
        }
        issued = n + 1;
      }
      for (int n = issued - SK_CSTAGES > 0 ? issued - SK_CSTAGES : 0; n < issued; ++n)
        mbar_wait(&cfull[n % SK_CSTAGES], (n / SK_CSTAGES) & 1, 2);
    }
  } else if (warp == 2) {
    if (lane == 0 && n_units > 0) {
      // ---------------- A-ring producer: LoRA weight tiles by TMA, else a plain arrival
      int done = 0;
      UnitCursor cur;
      cur.init(u0, S_t);
      for (int n = 0; n < n_units; ++n, cur.next()) {
        const int tile = cur.tile;
        const int k = cur.k;
        const int as = n % SK_ASTAGES;
        if (!mbar_wait(&aempty[as], ((n / SK_ASTAGES) & 1) ^ 1, 3)) break;
        if (k < p.k_stages) {
          mbar_arrive(&afull[as]);
        } else {
          mbar_arrive_expect_tx(&afull[as], SK_A_BYTES);
          tma_load_2d(sA + as * SK_A_BYTES, &tmL2x, &afull[as], (k - p.k_stages) * SK_BK, tile * SK_BN);
        }
        done = n + 1;
      }
      // No TMA load may still be in flight when the CTA exits: wait for the
      // final phase of each A slot (the last units' phases; earlier phases of a
      // slot must not be waited on, their parity repeats).
      for (int n = done - SK_ASTAGES > 0 ? done - SK_ASTAGES : 0; n < done; ++n)
        mbar_wait(&afull[n % SK_ASTAGES], (n / SK_ASTAGES) & 1, 4);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_units > 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16(128, p.nmma, false, false);
      int seg = -1;
      UnitCursor cur;
      cur.init(u0, S_t);
      for (int n = 0; n < n_units; ++n, cur.next()) {
        const int k = cur.k;
        const bool first = (n == 0) || (k == 0);
        const bool last = (n == n_units - 1) || (k == S_t - 1);
        if (first) {
          ++seg;
          if (seg >= 2 && !mbar_wait(&acce[seg & 1], ((seg >> 1) - 1) & 1, 5)) break;
        }
        const int cs = n % SK_CSTAGES;
        const int as = n % SK_ASTAGES;
        if (!mbar_wait(&cfull[cs], (n / SK_CSTAGES) & 1, 6)) break;
        if (!mbar_wait(&afull[as], (n / SK_ASTAGES) & 1, 7)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + as * SK_A_BYTES);
        const uint32_t b_base = smem_u32(sC + cs * SK_CSLOT);
        const uint32_t d = tmem + static_cast<uint32_t>(seg & 1) * 32u;
#pragma unroll
        for (int kk = 0; kk < SK_BK / 16; ++kk)
          umma_bf16(d, sw128_desc(a_base + kk * 32, 16, 1024), sw128_desc(b_base + kk * 32, 16, 1024), idesc,
                    (first && kk == 0) ? 0u : 1u);
        umma_commit(&cempty[cs]);
        umma_commit(&aempty[as]);
        if (last) umma_commit(&accf[seg & 1]);
      }
    }
  } else if (warp >= 4 && warp < SK_EPI_WARP0) {
    // ---------------- expanders: thread (e, part) owns elements
    // [16 part, 16 part + 16) of row tile * 128 + e of W^T
    const int e = (threadIdx.x - 128) & (SK_BN - 1);
    const int part = (threadIdx.x - 128) / SK_BN;
    const uint32_t qbase = smem_u32(s_q);
    const float mu = __ldg(p.dq_mean);
    ConstCache cc;
    // Block constants ride a register ring kPre units ahead of the expansion
    // (slot t of the ring serves units t, t + kPre, ...; the loop is unrolled
    // by kPre so every slot index is static), so their global-load latency is
    // covered by several units of work.
    constexpr int kPre = 6;
    uint32_t ec[kPre];
    float sc[kPre];
    UnitCursor cur, pf;
    cur.init(u0, S_t);
    pf.init(u0, S_t);
    auto fetch = [&](int n, uint32_t& e8, float& s32) {
      e8 = 0;
      s32 = 0.0f;
      if (n < n_units) {
        const int row = pf.tile * SK_BN + e;
        if (pf.k < p.k_stages && row < p.N) {
          const int64_t blk = static_cast<int64_t>(row) * p.blocks_per_row + pf.k;
          e8 = __ldg(p.absmax_fp8 + blk);
          s32 = __ldg(p.dq_scale + (blk >> 8));
        }
      }
      pf.next();
    };
#pragma unroll
    for (int t = 0; t < kPre; ++t) fetch(t, ec[t], sc[t]);
    bool ok = true;
    for (int n0 = 0; n0 < n_units && ok; n0 += kPre) {
#pragma unroll
      for (int t = 0; t < kPre; ++t) {
        const int n = n0 + t;
        if (n >= n_units || !ok) break;
        const int row = cur.tile * SK_BN + e;
        const int k = cur.k;
        const int cs = n % SK_CSTAGES;
        const int as = n % SK_ASTAGES;
        const uint32_t e_now = ec[t];
        const float s_now = sc[t];
        fetch(n + kPre, ec[t], sc[t]);
        if (k < p.k_stages) {
          const float cp = row < p.N ? cc.constant(static_cast<uint8_t>(e_now), s_now, mu) : 0.0f;
          if (!mbar_wait(&cfull[cs], (n / SK_CSTAGES) & 1, 8)) {
            ok = false;
            break;
          }
          constexpr int kWords = 8 / SK_SPLIT;  // 32-bit code words (8 elements each) per thread
          const uint32_t* codes = reinterpret_cast<const uint32_t*>(sC + cs * SK_CSLOT + SK_X_BYTES + e * 32) +
                                  part * kWords;
          uint32_t words[kWords];
#pragma unroll
          for (int c = 0; c < kWords; ++c) words[c] = codes[c];
          if (!mbar_wait(&aempty[as], ((n / SK_ASTAGES) & 1) ^ 1, 9)) {
            ok = false;
            break;
          }
          uint8_t* arow = sA + as * SK_A_BYTES + (e >> 3) * 1024 + (e & 7) * 128;
#pragma unroll
          for (int c = 0; c < kWords; ++c) {
            const int chunk = part * kWords + c;
            *reinterpret_cast<uint4*>(arow + ((chunk ^ (e & 7)) << 4)) = expand_word_smem(qbase, words[c], cp);
          }
          fence_proxy_async_smem();
        } else {
          if (!mbar_wait(&aempty[as], ((n / SK_ASTAGES) & 1) ^ 1, 10)) {
            ok = false;
            break;
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&afull[as]);
          mbar_arrive(&cempty[cs]);
        }
        cur.next();
      }
    }
  } else if (warp >= SK_EPI_WARP0) {
    // ---------------- epilogue: add each finished segment into Y
    const int q = warp & 3;
    int seg = -1;
    UnitCursor cur;
    cur.init(u0, S_t);
    for (int n = 0; n < n_units; ++n, cur.next()) {
      const int k = cur.k;
      if (n == 0 || k == 0) ++seg;
      const bool last = (n == n_units - 1) || (k == S_t - 1);
      if (!last) continue;
      const int buf = seg & 1;
      if (!mbar_wait(&accf[buf], (seg >> 1) & 1, 11)) break;
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
    tmem_dealloc(tmem, 64);
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
