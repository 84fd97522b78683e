// quant.cuh - NF4 blockwise quantization, double quantization of the block
// constants, and doubleDequant to bf16 (QLoRA; diycv.top walkthrough,
// "方法总览" §1-§3 and the doubleDequant equation of "关键公式").
//
// All three kernels stream HBM: one pass over the input, one over the output,
// 16-byte vector accesses, grid-stride loops sized in multiples of the SM count.
#pragma once

#include "common.cuh"


#include <cfloat>
#include <cmath>
#include <cstring>

namespace qlora {

// ====================================================================== host: decision table

// The quantizer's rule per element is code = #{j : fp32(w / c) > t_j}.  For a
// fixed absmax c the map w -> fp32(w / c) is monotone, so there is a largest
// bf16 value B_j(c) with fp32(B_j / c) <= t_j, and code = #{j : w > B_j(c)}:
// fifteen compares, no division.  For c = m 2^k, fp32(w / c) = fp32((w 2^-k) / m)
// whenever w 2^-k is exact, so a table over the 128 bf16 significands m in
// [1, 2) serves every normal absmax: the kernel scales the elements by 2^-k
// (elements that fall below the normal range are far from every boundary, so
// their rounding changes no compare) and compares them with row m.

static_assert(FLT_EVAL_METHOD == 0, "host float arithmetic must be IEEE single precision");

static inline float host_bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

static inline uint16_t host_float_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint32_t keep = u >> 16, low = u & 0xFFFFu;
  if (low > 0x8000u || (low == 0x8000u && (keep & 1u))) keep += 1;
  return static_cast<uint16_t>(keep);
}

// Total order on bf16 bit patterns that matches the order of their values
// (with -0 just below +0).
static inline int32_t bf16_key(uint16_t b) {
  return (b & 0x8000u) ? -static_cast<int32_t>(b & 0x7FFFu) - 1 : static_cast<int32_t>(b);
}
static inline uint16_t bf16_from_key(int32_t k) {
  return k >= 0 ? static_cast<uint16_t>(k) : static_cast<uint16_t>(0x8000u | static_cast<uint32_t>(-k - 1));
}

static inline float host_div_rn(float a, float b) {
  volatile float q = a / b;  // IEEE binary32 division, round to nearest even
  return q;
}

struct BoundaryTable {
  uint16_t b[128][16];  // bf16 bit patterns; entry 15 unused (0)
  int kmin, kmax;       // block exponents k (c = m * 2^k) the table covers exactly
  bool ok;              // every entry is a normal bf16
  bool bins_ok;         // every row's boundaries fall in distinct bins (host_bin)
};

// The quantizer's bin of a scaled element x (|x| < 2): the bf16 rounding of
// 31 x + 192, minus 128, in [2, 126].  The kernel computes it with one paired
// bf16 fused multiply-add (a single round-to-nearest-even of the exact value);
// here 31 x + 192 is exact in double and nearbyint rounds to nearest even.
// Bins are monotone in x and 1/31 wide.
static inline int host_bin(uint16_t xb) {
  const double v = 31.0 * static_cast<double>(host_bf16_to_float(xb)) + 192.0;
  return static_cast<int>(std::nearbyint(v)) - 128;
}

// Returns false if a search failed to converge (cannot happen for a valid
// codebook; kept as a guard).
static bool build_boundary_table(const float t[15], BoundaryTable* out) {
  int emin = 255, emax = 0;
  bool ok = true;
  for (int m = 0; m < 128; ++m) {
    const uint16_t cbits = static_cast<uint16_t>((127u << 7) | static_cast<uint32_t>(m));
    const float c = host_bf16_to_float(cbits);
    for (int j = 0; j < 15; ++j) {
      int32_t k = bf16_key(host_float_to_bf16_rne(t[j] * c));
      int steps = 0;
      while (host_div_rn(host_bf16_to_float(bf16_from_key(k)), c) > t[j]) {
        --k;
        if (++steps > 64) return false;
      }
      while (host_div_rn(host_bf16_to_float(bf16_from_key(k + 1)), c) <= t[j]) {
        ++k;
        if (++steps > 64) return false;
      }
      const uint16_t b = bf16_from_key(k);
      out->b[m][j] = b;
      const int e = (b >> 7) & 0xFF;
      if (e == 0 || e == 255) ok = false;
      emin = e < emin ? e : emin;
      emax = e > emax ? e : emax;
    }
    out->b[m][15] = 0;
  }
  out->ok = ok;
  // Each bin may hold at most one boundary, so that within a bin the code is
  // base or base + 1: the boundaries of every row must fall in strictly
  // increasing bins (they lie in (-2, 2) since |t_j| < 1 and m < 2).
  bool bins_ok = ok;
  for (int m = 0; m < 128 && bins_ok; ++m) {
    int prev = -1;
    for (int j = 0; j < 15; ++j) {
      const float v = host_bf16_to_float(out->b[m][j]);
      if (!(std::fabs(v) < 2.0f)) {
        bins_ok = false;
        break;
      }
      const int bin = host_bin(out->b[m][j]);
      if (bin <= prev) {
        bins_ok = false;
        break;
      }
      prev = bin;
    }
  }
  out->bins_ok = bins_ok;
  // Scaled entries keep a biased exponent in [1, 254]: e + k in that range.
  out->kmin = 1 - emin;
  out->kmax = 254 - emax;
  return true;
}

// ====================================================================== host: NF4 code values

// Standard normal quantile Q(p) for p in (0, 1): Newton's method on
// Phi(x) - p with Phi(x) = erfc(-x / sqrt 2) / 2 and Phi'(x) = exp(-x^2/2) / sqrt(2 pi),
// started from the logistic approximation x0 = log(p / (1 - p)) * sqrt(3) / pi.
static double normal_quantile(double p) {
  const double kPi = 3.14159265358979323846;
  double x = std::log(p / (1.0 - p)) * std::sqrt(3.0) / kPi;
  for (int it = 0; it < 100; ++it) {
    const double f = 0.5 * std::erfc(-x / std::sqrt(2.0)) - p;
    const double d = std::exp(-0.5 * x * x) / std::sqrt(2.0 * kPi);
    const double step = f / d;
    x -= step;
    if (std::fabs(step) <= 1e-17 * (1.0 + std::fabs(x))) break;
  }
  return x;
}

// The 16 NF4 code values (QLoRA NF4 data type): each half from standard-normal
// quantiles at evenly spaced probabilities between delta and 1/2 (9 points for
// the positive half, 8 for the negative half, the point 1/2 itself dropped),
// one exact zero, everything divided by the largest value.  delta is the
// midpoint of 1 - 1/30 and 1 - 1/32.
static void nf4_code_values(float out[16]) {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double v[16];
  int k = 0;
  // p_i = i * ((1/2 - delta) / (n - 1)) + delta, i = 0 .. n - 2 (the last point, 1/2, is dropped)
  const double step_neg = (0.5 - delta) / 7.0;
  const double step_pos = (0.5 - delta) / 8.0;
  for (int i = 0; i <= 6; ++i) v[k++] = -normal_quantile(static_cast<double>(i) * step_neg + delta);  // ascending
  v[k++] = 0.0;
  for (int i = 7; i >= 0; --i) v[k++] = normal_quantile(static_cast<double>(i) * step_pos + delta);   // ascending
  const double vmax = v[15];
  for (int j = 0; j < 16; ++j) out[j] = static_cast<float>(v[j] / vmax);
}

// Thresholds t_j = fp32((q_j + q_{j+1}) / 2): the fp64 sum of two fp32 values
// and the halving are exact, then one rounding to fp32.
static inline void nf4_thresholds(const float q[16], float t[15]) {
  for (int j = 0; j < 15; ++j) t[j] = static_cast<float>((static_cast<double>(q[j]) + q[j + 1]) / 2.0);
}

// ====================================================================== K1: quantize

struct QuantizeParams {
  const uint4* w;        // bf16 input viewed as 16-byte vectors
  uint2* codes;          // 8 code bytes (16 codes) per thread-quarter
  float* absmax;
  int64_t nblocks;
  float t[16];           // t[0..14] thresholds
  uint32_t zero_code;
  uint32_t fast_ok;      // every table entry is a normal bf16
  uint32_t bin_ok;       // and the boundaries of every row fall in distinct bins
  uint32_t bnd[128][16];  // boundary B_j(m) as bf16, duplicated into both halves
};

// ---- bin path (bin_ok): one lookup per element instead of a 4-level search.
// Scaled element x (|x| < 2) -> bin = bf16(31 x + 192) - 128 (the low byte of
// the bf16 result, whose binade [128, 256) has a zero exponent LSB).  Every
// bin holds at most one boundary of row m, so within a bin the code is
// base(m, bin) + [x > thr(m, bin)].  The shared table holds, per (m, bin), the
// word {lo: bf16(128 + base), hi: thr as bf16} (thr = +inf where the bin has
// no boundary that an element of the bin can exceed).  Per element pair: one
// paired bf16 multiply-add (bins), two 4-byte lookups, two byte permutes, one
// paired compare (1.0 / 0.0) and one paired add, which leaves bf16(128 + code)
// whose low byte is the code.
constexpr int kQuantBinSmem = 128 * 128 * 4;
constexpr uint32_t kBinMul2 = 0x41F841F8u;  // bf16x2 {31, 31}
constexpr uint32_t kBinAdd2 = 0x43404340u;  // bf16x2 {192, 192}

__device__ __forceinline__ uint32_t bin_pair(uint32_t x2) {
  const uint32_t mul = kBinMul2, add = kBinAdd2;
  const __nv_bfloat162 r = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&x2),
                                   *reinterpret_cast<const __nv_bfloat162*>(&mul),
                                   *reinterpret_cast<const __nv_bfloat162*>(&add));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Builds the (m, bin) table from the boundary rows: warp w takes rows w, w + 8,
// ...; lane j < 15 bins boundary j (and its bf16 successor, to know whether an
// element of the same bin can exceed it); the bins holding a boundary form a
// 128-bit map, and bin b's base is the number of boundaries in lower bins.
__device__ __forceinline__ void build_bin_table(uint32_t* tab, const uint32_t* bnd /* [128][16] in smem */) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int m = warp; m < 128; m += blockDim.x >> 5) {
    uint32_t bj = 0, binj = 0;
    bool has = false, exceedable = false;
    if (lane < 15) {
      bj = bnd[m * 16 + lane] & 0xFFFFu;
      // successor in value order (boundaries are never zero)
      const uint32_t nb = (bj & 0x8000u) ? bj - 1u : bj + 1u;
      binj = bin_pair(bj * 0x00010001u) & 0x7Fu;
      exceedable = (bin_pair(nb * 0x00010001u) & 0x7Fu) == binj;
      has = true;
    }
    uint32_t occ[4], exc[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const bool here = has && (binj >> 5) == static_cast<uint32_t>(w);
      occ[w] = __reduce_or_sync(0xFFFFFFFFu, here ? 1u << (binj & 31u) : 0u);
      exc[w] = __reduce_or_sync(0xFFFFFFFFu, here && exceedable ? 1u << (binj & 31u) : 0u);
    }
    uint32_t below = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t base = below + __popc(occ[w] & ((1u << lane) - 1u));
      below += __popc(occ[w]);
      const uint32_t thr_b = __shfl_sync(0xFFFFFFFFu, bj, static_cast<int>(base & 15u));
      const uint32_t thr = ((exc[w] >> lane) & 1u) ? thr_b : 0x7F80u;
      tab[m * 128 + 32 * w + lane] = (thr << 16) | (0x4300u + base);
    }
  }
}

__device__ __forceinline__ uint32_t bf16x2_gt_mask(uint32_t a, uint32_t b) {
  return __hgt2_mask(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
}

__device__ __forceinline__ uint32_t sel_mask(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

// Codes of the two bf16 elements of a packed pair (scaled by 2^-k) by
// a 4-level binary search over the sorted boundaries B[0..14].  Returns
// element 0's code in bits 4..7 and element 1's in bits 16..19.
__device__ __forceinline__ uint32_t code_pair(uint32_t w2, const uint32_t (&B)[16]) {
  const uint32_t m1 = bf16x2_gt_mask(w2, B[7]);
  const uint32_t m2 = bf16x2_gt_mask(w2, sel_mask(m1, B[11], B[3]));
  const uint32_t t3 = sel_mask(m1, sel_mask(m2, B[13], B[9]), sel_mask(m2, B[5], B[1]));
  const uint32_t m3 = bf16x2_gt_mask(w2, t3);
  const uint32_t t4 = sel_mask(m1, sel_mask(m2, sel_mask(m3, B[14], B[12]), sel_mask(m3, B[10], B[8])),
                               sel_mask(m2, sel_mask(m3, B[6], B[4]), sel_mask(m3, B[2], B[0])));
  const uint32_t m4 = bf16x2_gt_mask(w2, t4);
  return (m1 & 0x00080080u) | (m2 & 0x00040040u) | (m3 & 0x00020020u) | (m4 & 0x00010010u);
}

__device__ __forceinline__ uint32_t pair_byte(uint32_t acc) { return (acc | (acc >> 16)) & 0xFFu; }

// Codes of the 16 elements w[0..7] (bf16 pairs) of one lane, whose block has
// absmax bits cbits; returns 8 packed code bytes.  For a normal absmax
// c = m 2^k with |k| <= 126 the elements are scaled by 2^-k, which is exact
// (results below the normal range only meet boundaries far from zero, so
// their rounding changes no comparison), and compared with the boundaries of
// the table row of the significand m.
__device__ __forceinline__ uint2 quantize16(const QuantizeParams& p, const uint4 (*s_bnd)[4], const uint32_t* s_tab,
                                            const uint32_t (&w)[8], uint32_t cbits) {
  const uint32_t exp_c = cbits >> 7;
  uint2 out;
  if (cbits == 0) {
    const uint32_t z = ((p.zero_code << 4) | p.zero_code) * 0x01010101u;
    out.x = z;
    out.y = z;
  } else if (p.bin_ok && exp_c >= 1 && exp_c <= 253) {
    const uint32_t* row = s_tab + ((cbits & 0x7Fu) << 7);
    const uint32_t sb2 = ((254u - exp_c) << 7) * 0x00010001u;  // bf16x2 2^-k
    const __nv_bfloat162 scale = *reinterpret_cast<const __nv_bfloat162*>(&sb2);
    uint32_t c2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 x = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]), scale);
      const uint32_t y = bin_pair(*reinterpret_cast<const uint32_t*>(&x));
      const uint32_t e0 = row[y & 0x7Fu], e1 = row[(y >> 16) & 0x7Fu];
      const uint32_t thr = __byte_perm(e0, e1, 0x7632), base = __byte_perm(e0, e1, 0x5410);
      const __nv_bfloat162 code = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&base),
                                          __hgt2(x, *reinterpret_cast<const __nv_bfloat162*>(&thr)));
      c2[i] = *reinterpret_cast<const uint32_t*>(&code);  // bytes 0 / 2: codes of elements 2i / 2i + 1
    }
    uint32_t o2[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t a = __byte_perm(c2[4 * q], c2[4 * q + 1], 0x6240);
      const uint32_t b = __byte_perm(c2[4 * q + 2], c2[4 * q + 3], 0x6240);
      // high nibbles (even elements) * 16 + low nibbles (odd elements), byte-wise without carries
      o2[q] = __byte_perm(a, b, 0x5410) * 16u + __byte_perm(a, b, 0x7632);
    }
    out.x = o2[0];
    out.y = o2[1];
  } else if (p.fast_ok && exp_c >= 1 && exp_c <= 253) {
    uint32_t B[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 t = s_bnd[cbits & 0x7Fu][q];
      B[4 * q + 0] = t.x;
      B[4 * q + 1] = t.y;
      B[4 * q + 2] = t.z;
      B[4 * q + 3] = t.w;
    }
    const uint32_t sb2 = ((254u - exp_c) << 7) * 0x00010001u;  // bf16x2 2^-k
    const __nv_bfloat162 scale = *reinterpret_cast<const __nv_bfloat162*>(&sb2);
    uint32_t bytes[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 x = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]), scale);
      bytes[i] = pair_byte(code_pair(*reinterpret_cast<const uint32_t*>(&x), B));
    }
    out.x = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
    out.y = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
  } else {
    // Exact rule by division: absmax subnormal or in the top binade, or a
    // codebook whose boundaries are not all normal.
    const float c = bf16_bits_to_float(cbits);
    uint32_t bytes[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t cc[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float x = __fdiv_rn(bf16_bits_to_float((w[i] >> (16 * h)) & 0xFFFFu), c);
        uint32_t code = 0;
#pragma unroll
        for (int j = 0; j < 15; ++j) code += (x > p.t[j]) ? 1u : 0u;
        cc[h] = code;
      }
      bytes[i] = (cc[0] << 4) | cc[1];
    }
    out.x = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
    out.y = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
  }
  return out;
}

// absmax bits of the block shared by each group of 4 lanes (|bf16| bit order
// is value order for non-negative values).
__device__ __forceinline__ uint32_t block_absmax_bits(const uint32_t (&w)[8]) {
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
  uint32_t cbits = max(mx & 0xFFFFu, mx >> 16);
  cbits = max(cbits, __shfl_xor_sync(0xFFFFFFFFu, cbits, 1));
  cbits = max(cbits, __shfl_xor_sync(0xFFFFFFFFu, cbits, 2));
  return cbits;
}

// Each group of 4 lanes owns one 64-element block (16 elements per lane); a
// warp takes 16 blocks (2 KB of input, two independent halves) per iteration.
// The grid is a few CTAs per SM and loops over the tensor.
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const __grid_constant__ QuantizeParams p) {
  __shared__ uint4 s_bnd[128][4];
  extern __shared__ uint32_t s_tab[];  // 128 x 128 bin table (kQuantBinSmem bytes) when p.bin_ok
  {
    const uint4* src = reinterpret_cast<const uint4*>(&p.bnd[0][0]);
    for (int i = threadIdx.x; i < 128 * 4; i += blockDim.x) s_bnd[i >> 2][i & 3] = src[i];
  }
  __syncthreads();
  if (p.bin_ok) {
    build_bin_table(s_tab, reinterpret_cast<const uint32_t*>(&s_bnd[0][0]));
    __syncthreads();
  }

  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);

  for (int64_t b0 = warp_global * 16; b0 < p.nblocks; b0 += warp_stride * 16) {
    const int64_t blk0 = b0 + (lane >> 2);
    const int64_t blk1 = blk0 + 8;
    const bool v0ok = blk0 < p.nblocks, v1ok = blk1 < p.nblocks;
    uint4 a0 = make_uint4(0, 0, 0, 0), a1 = a0, b0v = a0, b1v = a0;
    if (v0ok) {
      const uint4* src = p.w + blk0 * 8 + sub * 2;
      a0 = __ldcs(src);
      a1 = __ldcs(src + 1);
    }
    if (v1ok) {
      const uint4* src = p.w + blk1 * 8 + sub * 2;
      b0v = __ldcs(src);
      b1v = __ldcs(src + 1);
    }
    const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const uint32_t wb[8] = {b0v.x, b0v.y, b0v.z, b0v.w, b1v.x, b1v.y, b1v.z, b1v.w};
    const uint32_t ca = block_absmax_bits(wa);
    const uint32_t cb = block_absmax_bits(wb);
    if (sub == 0) {
      if (v0ok) p.absmax[blk0] = bf16_bits_to_float(ca);
      if (v1ok) p.absmax[blk1] = bf16_bits_to_float(cb);
    }
    const uint2 oa = quantize16(p, s_bnd, s_tab, wa, ca);
    const uint2 ob = quantize16(p, s_bnd, s_tab, wb, cb);
    if (v0ok) __stcs(p.codes + blk0 * 4 + sub, oa);
    if (v1ok) __stcs(p.codes + blk1 * 4 + sub, ob);
  }
}

// ====================================================================== K2: double quantization

// Pass 1: exact fp64 sum of all block constants (one atomic per CTA).  Every
// constant is a bf16 value, so while the total fits in 53 bits every partial
// sum is exact and the order of the additions does not matter.
__global__ void __launch_bounds__(256) dq_sum_kernel(const float4* __restrict__ absmax4, int64_t n4,
                                                     double* __restrict__ sum) {
  __shared__ double s_part[8];
  double acc = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(absmax4 + i);
    acc += static_cast<double>(v.x);
    acc += static_cast<double>(v.y);
    acc += static_cast<double>(v.z);
    acc += static_cast<double>(v.w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (blockDim.x >> 5); ++i) t += s_part[i];
    if (t != 0.0) atomicAdd(sum, t);
  }
}

// Pass 2: one warp per group of 256 constants.  mu = fp32(sum / nb);
// d = fp32(c - mu); dq_scale = max |d|; code = E4M3(fp32(d * fp32(448 / dq_scale))).
__global__ void __launch_bounds__(256) dq_encode_kernel(const float4* __restrict__ absmax4, int64_t ngroups,
                                                        int64_t nblocks, const double* __restrict__ sum,
                                                        uint2* __restrict__ fp8_out, float* __restrict__ dq_scale,
                                                        float* __restrict__ dq_mean) {
  const double total = *sum;
  const float mu = __double2float_rn(__ddiv_rn(total, static_cast<double>(nblocks)));
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  if (warp_global == 0 && lane == 0) *dq_mean = mu;
  for (int64_t g = warp_global; g < ngroups; g += warp_stride) {
    const float4 a = __ldg(absmax4 + g * 64 + lane * 2);
    const float4 b = __ldg(absmax4 + g * 64 + lane * 2 + 1);
    float d[8] = {__fsub_rn(a.x, mu), __fsub_rn(a.y, mu), __fsub_rn(a.z, mu), __fsub_rn(a.w, mu),
                  __fsub_rn(b.x, mu), __fsub_rn(b.y, mu), __fsub_rn(b.z, mu), __fsub_rn(b.w, mu)};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(d[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    uint32_t e[8];
    if (m > 0.0f) {
      const float inv = __fdiv_rn(448.0f, m);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        e[i] = static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fmul_rn(d[i], inv), __NV_SATFINITE, __NV_E4M3));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) e[i] = 0u;
    }
    uint2 out;
    out.x = e[0] | (e[1] << 8) | (e[2] << 16) | (e[3] << 24);
    out.y = e[4] | (e[5] << 8) | (e[6] << 16) | (e[7] << 24);
    fp8_out[g * 32 + lane] = out;
    if (lane == 0) dq_scale[g] = m;
  }
}

// ====================================================================== K3: dequant

struct DequantParams {
  const uint32_t* codes;    // 8 codes per 32-bit word
  const uint8_t* absmax_fp8;
  const float* dq_scale;
  const float* dq_mean;
  const float* absmax32;    // single-level constants (no double quantization), or null
  uint4* out;               // bf16 output, 8 per 16 bytes
  int64_t nwords;           // n / 8
  int64_t nblocks;          // n / 64
  float codebook[16];
};

constexpr int kDequantThreads = 1024;
constexpr int kDequantWords = 8;  // code words per lane per step
// The pair table needs a 64 KB-aligned window address inside dynamic shared
// memory: 128 KB always holds one.
constexpr int kDequantSmem = 2 * static_cast<int>(kPairTabBytes);

// A warp step covers 256 consecutive code words (32 blocks, 8 KB of bf16):
// in sub-step u lane l expands word 32 u + l, so each warp store writes 512
// contiguous bytes.  Lane l first computes the constant c' of the step's
// block l; the word's constant then comes by one shuffle.  Each code byte
// costs one byte permute, one conflict-free 8-byte lookup in the pair table,
// one paired fp32 multiply by c' and one paired rounding to bf16.  One CTA of
// 1024 threads per SM, grid-stride over the tensor.
__global__ void __launch_bounds__(kDequantThreads, 1) nf4_dequant_kernel(const __grid_constant__ DequantParams p) {
  extern __shared__ __align__(16) uint8_t dsmem[];
  const uint32_t toff = pair_tab_offset(dsmem);
  if (toff + kPairTabBytes > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusSmemLayout);
    return;
  }
  uint8_t* tab = dsmem + toff;
  fill_pair_table(tab, p.codebook);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t key = pair_key(tab, lane);
  const float mu = p.absmax32 ? 0.0f : __ldg(p.dq_mean);
  ConstCache cc;
  constexpr int kStepWords = 32 * kDequantWords;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t wb = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kStepWords;
       wb < p.nwords; wb += nwarps * kStepWords) {
    uint32_t w[kDequantWords];
#pragma unroll
    for (int u = 0; u < kDequantWords; ++u) {
      const int64_t i = wb + u * 32 + lane;
      w[u] = i < p.nwords ? __ldcs(p.codes + i) : 0u;
    }
    const int64_t blk = (wb >> 3) + lane;
    float cp = 0.0f;
    if (blk < p.nblocks)
      cp = p.absmax32 ? __ldg(p.absmax32 + blk) : cc.constant(__ldg(p.absmax_fp8 + blk), __ldg(p.dq_scale + (blk >> 8)), mu);
#pragma unroll
    for (int u = 0; u < kDequantWords; ++u) {
      const int64_t i = wb + u * 32 + lane;
      const float c = __shfl_sync(0xFFFFFFFFu, cp, u * 4 + (lane >> 3));
      if (i < p.nwords) __stcs(p.out + i, word_dequant(w[u], key, dup_f32x2(c)));
    }
  }
}

}  // namespace qlora
