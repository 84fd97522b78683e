// gemm.cuh - tcgen05 (5th-generation tensor core) GEMMs of the QLoRA linear
// layer (diycv.top walkthrough, "关键公式": Y = X doubleDequant(c1, c2, W)
// + s X L1 L2; "训练" step 5 for the backward products).
//
// qgemm_nf4_kernel : D = A * W'(op) + A_ext * B_ext, W' dequantized on the fly.
//   Forward  (Y  = X  W'   + [sT_hi|sT_lo] [L2;L2]) : W' operand K-major.
//   Backward (dX = dY W'^T + [sU_hi|sU_lo] [L1;L1]^T): W' operand MN-major.
//   Warp roles (384 threads): warp 0 lane 0 issues TMA loads of the A tiles
//   (and of the LoRA tiles), warp 1 lane 0 issues tcgen05.mma, warps 4..11
//   ("expanders") read packed NF4 codes from HBM, build a per-block 16-entry
//   bf16 table and write the dequantized tile straight into the swizzled
//   shared-memory layout the tensor core reads; warps 0..3 drain TMEM.
//   Tile 256 x 256 x 64: two M=128 MMAs share every dequantized B tile, which
//   halves the dequantization work per flop.
//
// gemm_tma_kernel  : D (+)= A * (B [+ B2]) for the rank-r products
//   T = X L1, U = dY L2^T, dL1 = X^T (sU), dL2^T = dY^T (sT), with split-K
//   over the long reduction and fp32 atomic accumulation.
#pragma once

#include "common.cuh"

namespace qlora {

// ====================================================================== fused NF4 GEMM

constexpr int QG_BM = 256;
constexpr int QG_BN = 256;
constexpr int QG_BK = 64;
constexpr int QG_STAGES = 3;
constexpr int QG_THREADS = 384;
constexpr int QG_TILE_BYTES = 256 * 64 * 2;  // one A or B stage: 32 KB
constexpr int QG_LUT_BYTES = 16 * 256 * 4;   // 16 entries x 256 expander threads, u32 slots
// LUT (16 KB-aligned) | A[3] | B[3] | barriers; plus up to 15 KB of alignment slack.
constexpr int QG_SMEM_USED = QG_LUT_BYTES + 2 * QG_STAGES * QG_TILE_BYTES + 256;
constexpr int QG_SMEM_BYTES = QG_SMEM_USED + 16384;

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
                     const __grid_constant__ CUtensorMap tmBe, const uint8_t* __restrict__ codes,
                     const __grid_constant__ QGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t lut_u32 = (raw_u32 + 16383u) & ~16383u;
  uint8_t* lut = smem_raw + (lut_u32 - raw_u32);
  uint8_t* sA = lut + QG_LUT_BYTES;
  uint8_t* sB = sA + QG_STAGES * QG_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + QG_STAGES * QG_TILE_BYTES);
  uint64_t* full_a = bars;                 // TMA bytes of A (and B on LoRA stages)
  uint64_t* full_b = bars + QG_STAGES;     // 8 expander warps
  uint64_t* empty = bars + 2 * QG_STAGES;  // tcgen05.commit
  uint64_t* accum = bars + 3 * QG_STAGES;  // last MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * QG_STAGES + 1);

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
    mbar_init(accum, 1);
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmAe);
    tma_prefetch_map(&tmBe);
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
      // ---------------- TMA producer
      int issued = 0;
      for (int i = 0; i < S; ++i) {
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
      // Leave no copy in flight: wait (bounded) for the last load of each slot.
      for (int i = issued - QG_STAGES > 0 ? issued - QG_STAGES : 0; i < issued; ++i)
        mbar_wait(&full_a[i % QG_STAGES], (i / QG_STAGES) & 1);
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
    // ---------------- expanders: 256 threads, one (row, 64-block) each per stage
    const int e = threadIdx.x - 128;
    const uint32_t my_lut = lut_u32 + static_cast<uint32_t>(e) * 4u;
    const float mu = __ldg(p.dq_mean);
    // Which 64-block of the stored W^T[o][h] this thread expands at stage i:
    //   forward : row n0 + e of W^T, block column i;
    //   backward: row 64 i + e / 4 of W^T, block column n0 / 64 + e % 4.
    const bool in_range = kBwd ? (n0 / 64 + (e & 3) < p.blocks_per_row) : (n0 + e < p.N);
    auto block_index = [&](int i) -> int64_t {
      return kBwd ? static_cast<int64_t>(i * 64 + (e >> 2)) * p.blocks_per_row + (n0 >> 6) + (e & 3)
                  : static_cast<int64_t>(n0 + e) * p.blocks_per_row + i;
    };
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    uint32_t ecode = 0;
    float scale = 0.0f;
    if (in_range && KM > 0) {
      const int64_t blk = block_index(0);
      const uint4* src = reinterpret_cast<const uint4*>(codes + blk * 32);
      c0 = __ldg(src);
      c1 = __ldg(src + 1);
      ecode = __ldg(p.absmax_fp8 + blk);
      scale = __ldg(p.dq_scale + (blk >> 8));
    }
    for (int i = 0; i < KM; ++i) {
      const int s = i % QG_STAGES;
      const uint32_t ph = (i / QG_STAGES) & 1;
      // prefetch the next stage's codes and constants
      uint4 n0c = make_uint4(0, 0, 0, 0), n1c = n0c;
      uint32_t necode = 0;
      float nscale = 0.0f;
      if (in_range && i + 1 < KM) {
        const int64_t blk = block_index(i + 1);
        const uint4* src = reinterpret_cast<const uint4*>(codes + blk * 32);
        n0c = __ldg(src);
        n1c = __ldg(src + 1);
        necode = __ldg(p.absmax_fp8 + blk);
        nscale = __ldg(p.dq_scale + (blk >> 8));
      }
      // 16-entry table of this block: bf16(q_j * c')
      const float cp = in_range ? block_constant(static_cast<uint8_t>(ecode), scale, mu) : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v = __fmul_rn(p.codebook[j], cp);
        const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(my_lut + j * 1024u), "r"(b) : "memory");
      }
      if (!mbar_wait(&empty[s], ph ^ 1)) break;
      uint8_t* bdst = sB + s * QG_TILE_BYTES;
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t wv = words[c];
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          // high nibble of byte b -> element 2b (low half), low nibble -> 2b + 1
          const uint32_t a_hi = ((wv >> (8 * b + 4)) & 0xFu) * 1024u + my_lut;
          const uint32_t a_lo = ((wv >> (8 * b)) & 0xFu) * 1024u + my_lut;
          uint32_t vh, vl;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(vh) : "r"(a_hi));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(vl) : "r"(a_lo));
          o[b] = vh | (vl << 16);
        }
        uint32_t off;
        if (kBwd) {
          const int kr = e >> 2;
          off = (e & 3) * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128 + ((c ^ (kr & 7)) << 4);
        } else {
          off = (e >> 3) * 1024 + (e & 7) * 128 + ((c ^ (e & 7)) << 4);
        }
        *reinterpret_cast<uint4*>(bdst + off) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_b[s]);
      c0 = n0c;
      c1 = n1c;
      ecode = necode;
      scale = nscale;
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
