// optim.cuh - the optimizer step of the LoRA factors (the only trained
// parameters; walkthrough "训练" step 6: the optimizer updates only the LoRA
// parameters, and the paged optimizer keeps its state in unified memory that
// moves to host RAM under memory pressure).
//
// AdamW with decoupled weight decay and global-norm gradient clipping (the
// recipe paragraph: Adam beta2 = 0.999, max grad norm 0.3, constant learning
// rate).  Both kernels stream HBM: the state may live in unified (managed)
// memory, in which case the first touch of a page that was moved to the host
// migrates it back.
#pragma once

#include "common.cuh"

namespace qlora {

// sum of g^2 over a flat fp32 array, added to *acc (fp64; one atomic per CTA).
__global__ void __launch_bounds__(256) grad_sqnorm_kernel(const float* __restrict__ g, int64_t n,
                                                          double* __restrict__ acc) {
  __shared__ double part[8];
  double s = 0.0;
  const int64_t n4 = n / 4;
  const bool vec = (reinterpret_cast<uintptr_t>(g) & 15u) == 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (vec) {
    for (int64_t i = tid; i < n4; i += stride) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(g) + i);
      s += static_cast<double>(v.x) * v.x + static_cast<double>(v.y) * v.y + static_cast<double>(v.z) * v.z +
           static_cast<double>(v.w) * v.w;
    }
    for (int64_t i = 4 * n4 + tid; i < n; i += stride) s += static_cast<double>(g[i]) * g[i];
  } else {
    for (int64_t i = tid; i < n; i += stride) s += static_cast<double>(g[i]) * g[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (blockDim.x >> 5); ++i) t += part[i];
    if (t != 0.0) atomicAdd(acc, t);
  }
}

struct AdamWParams {
  float lr, beta1, beta2, eps, weight_decay;
  float step_size;          // lr / (1 - beta1^t)
  float bc2_sqrt;           // sqrt(1 - beta2^t)
  float max_grad_norm;      // clipping threshold (used when sqnorm is given)
  const double* sqnorm;     // sum of squares of all gradients, or null (no clipping)
};

// One AdamW step per element, in the order of the usual formulation:
//   g <- g * min(1, max_norm / (||g|| + 1e-6))        (when clipping)
//   p <- p * (1 - lr wd)
//   m <- m + (1 - b1) (g - m)
//   v <- b2 v + (1 - b2) g^2
//   p <- p - step_size * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// fp32 IEEE arithmetic throughout; pb (optional) receives bf16(p), the copy
// the linear layer reads.
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    uint16_t* __restrict__ pb, int64_t n, AdamWParams a) {
  float clip = 1.0f;
  if (a.sqnorm) {
    const double norm = sqrt(*a.sqnorm);
    const float coef = static_cast<float>(static_cast<double>(a.max_grad_norm) / (norm + 1e-6));
    clip = coef < 1.0f ? coef : 1.0f;
  }
  const float decay = __fsub_rn(1.0f, __fmul_rn(a.lr, a.weight_decay));
  const float one_m_b1 = __fsub_rn(1.0f, a.beta1), one_m_b2 = __fsub_rn(1.0f, a.beta2);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float gi = a.sqnorm ? __fmul_rn(g[i], clip) : g[i];
    float pi = __fmul_rn(p[i], decay);
    const float mi = __fadd_rn(m[i], __fmul_rn(one_m_b1, __fsub_rn(gi, m[i])));
    const float vi = __fadd_rn(__fmul_rn(a.beta2, v[i]), __fmul_rn(one_m_b2, __fmul_rn(gi, gi)));
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(vi), a.bc2_sqrt), a.eps);
    pi = __fsub_rn(pi, __fmul_rn(a.step_size, __fdiv_rn(mi, denom)));
    p[i] = pi;
    m[i] = mi;
    v[i] = vi;
    if (pb) pb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pi));
  }
}

}  // namespace qlora
