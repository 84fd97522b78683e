// common.cuh - sm_100a building blocks shared by the QLoRA kernels:
// mbarriers with bounded waits, TMA tile loads (no multicast), tcgen05 MMA /
// TMEM helpers and the shared-memory matrix descriptors.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

// Device status word: bit 0 = a pipeline wait gave up (bit 1: see below).
// Read and cleared by qlora_check_status().  g_wait_tags records which waits
// gave up (one bit per call-site tag), for qlora_debug_wait_tags().
__device__ unsigned int g_status;
__device__ unsigned int g_wait_tags;

constexpr unsigned int kStatusTimeout = 1u;
// Bit 1: a kernel found its shared-memory layout impossible (the 64 KB-aligned
// pair table did not fit in the dynamic shared memory it was given) and did
// nothing.
constexpr unsigned int kStatusSmemLayout = 2u;
// A wait that has not completed after this many nanoseconds gives up.
constexpr unsigned long long kWaitLimitNs = 4000000000ull;
// Wait-site tag of the failure-path probe (qlora_debug_wait_probe).
constexpr int kTagWaitProbe = 30;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_count(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after
// limit_ns (kWaitLimitNs in every pipeline), records the timeout in g_status
// (and the call site's tag in g_wait_tags) and returns false, so that a broken
// pipeline ends the kernel instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int tag = 31,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (global_timer_ns() - t0 > limit_ns) {
        atomicOr(&g_status, kStatusTimeout);
        atomicOr(&g_wait_tags, 1u << (tag & 31));
        return false;
      }
    }
  }
}

// Like mbar_wait, for waits expected to be long (e.g. an epilogue waiting for a
// whole main loop): sleeps between polls so that the waiting warp does not
// take issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, int tag = 31) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(256);
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 15u) {
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_status, kStatusTimeout);
        atomicOr(&g_wait_tags, 1u << (tag & 31));
        return false;
      }
    }
  }
}

// mbar_wait by every lane of a warp with one warp-wide outcome, so that the
// warp stays converged for the .sync.aligned instructions that follow.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int tag = 31) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, tag));
}

__device__ __forceinline__ bool warp_wait_sleep(uint64_t* bar, uint32_t parity, int tag = 31) {
  return __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar, parity, tag));
}

// ------------------------------------------------------------------ TMA (tile mode, no multicast)

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Untiled bulk copy global -> shared of `bytes` bytes (both addresses 16-byte
// aligned, bytes a multiple of 16), completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulation, with the
// A operand read from tensor memory: row m of the 128-row tile in lane m, its
// K values packed two bf16 per 32-bit column (even k in the low half), so a
// K16 step spans 8 columns.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Non-blocking test of 12 barrier phases at once: all tests go out before any
// result is read, so the batch costs one shared-memory round trip.  (After
// tcgen05.mma instructions a thread's shared-memory accesses complete only
// after a long delay, ~0.1 us measured, so a thread that issues MMAs should
// read shared memory rarely and in batches.)  Returns 1 iff all complete.
__device__ __forceinline__ uint32_t mbar_test12(const uint32_t (&bar)[12], const uint32_t (&par)[12]) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p<12>;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p0, [%1], %13;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p1, [%2], %14;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p2, [%3], %15;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p3, [%4], %16;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p4, [%5], %17;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p5, [%6], %18;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p6, [%7], %19;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p7, [%8], %20;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p8, [%9], %21;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p9, [%10], %22;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p10, [%11], %23;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p11, [%12], %24;\n\t"
      "and.pred p0, p0, p1;\n\tand.pred p2, p2, p3;\n\tand.pred p4, p4, p5;\n\t"
      "and.pred p6, p6, p7;\n\tand.pred p8, p8, p9;\n\tand.pred p10, p10, p11;\n\t"
      "and.pred p0, p0, p2;\n\tand.pred p4, p4, p6;\n\tand.pred p8, p8, p10;\n\t"
      "and.pred p0, p0, p4;\n\tand.pred p0, p0, p8;\n\t"
      "selp.u32 %0, 1, 0, p0;\n\t}"
      : "=r"(ok)
      : "r"(bar[0]), "r"(bar[1]), "r"(bar[2]), "r"(bar[3]), "r"(bar[4]), "r"(bar[5]), "r"(bar[6]), "r"(bar[7]),
        "r"(bar[8]), "r"(bar[9]), "r"(bar[10]), "r"(bar[11]), "r"(par[0]), "r"(par[1]), "r"(par[2]), "r"(par[3]),
        "r"(par[4]), "r"(par[5]), "r"(par[6]), "r"(par[7]), "r"(par[8]), "r"(par[9]), "r"(par[10]), "r"(par[11])
      : "memory");
  return ok;
}

// Arrives on `bar` once every previously issued tcgen05.mma of this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Each thread of the warp reads 16 consecutive fp32 columns of its own TMEM
// lane (lane = 32 * (warp % 4) + laneid, given by the address).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Each thread of the warp writes 16 consecutive 32-bit columns of its own
// TMEM lane (lane = 32 * (warp % 4) + laneid, given by the address).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version 1).
//   K-major operand : rows of 128 B (64 bf16 along K), 8-row atoms of 1 KB;
//                     sbo = stride between 8-row atoms, lbo unused (16).
//   MN-major operand: 64 bf16 along M/N per 128-B row, 8 K-rows per 1-KB atom;
//                     lbo = stride between 64-wide M/N atoms,
//                     sbo = stride between 8-row K groups.
// The start address must lie in a 1024-byte-aligned swizzle atom; advancing
// K inside a K-major atom adds 32 B per 16 bf16.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for tcgen05
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 x bf16 -> fp32.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                  // D format fp32
         | (1u << 7)                                // A format bf16
         | (1u << 10)                               // B format bf16
         | ((a_mn_major ? 1u : 0u) << 15)           // A major
         | ((b_mn_major ? 1u : 0u) << 16)           // B major
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even, each half
  return *reinterpret_cast<uint32_t*>(&v);
}

// E4M3 code -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_float(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// 4 * (the 4-bit field of w at bit `pos`), a byte offset into a 16-entry fp32
// table.  The right shift is done as a high multiply (FMA pipe), leaving one
// logic op on the integer pipe.
__device__ __forceinline__ uint32_t nibble_x4(uint32_t w, int pos) {
  if (pos < 2) return (w << (2 - pos)) & 0x3Cu;
  return __umulhi(w, 1u << (34 - pos)) & 0x3Cu;
}

// Inner dequant of doubleDequant: the block constant
// c' = fp32(fp32(E4M3(e) * fp32(dq_scale / 448)) + mu), three separately
// rounded operations (no fused multiply-add).
__device__ __forceinline__ float block_constant(uint8_t e, float dq_scale, float mu) {
  return __fadd_rn(__fmul_rn(e4m3_to_float(e), __fdiv_rn(dq_scale, 448.0f)), mu);
}

// ====================================================================== register lookup table

// The 16 values bf16(q_j * c') of one block held in 8 registers: byte k of
// lo[i] / hi[i] is the low / high byte of entry 4 i + k.  Four codes are
// looked up at once with byte permutes (no shared memory, no divergence).
struct Lut16 {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ void build_lut16(const float (&q)[16], float cp, Lut16& L) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = pack_bf16x2(__fmul_rn(q[2 * i], cp), __fmul_rn(q[2 * i + 1], cp));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    L.lo[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x6420);
    L.hi[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x7531);
  }
}

// Dequantizes the 4 codes in the low 16 bits of g (two packed bytes; element
// 2k in the high nibble of byte k) to two bf16x2 words in element order.
__device__ __forceinline__ void lut_lookup4(const Lut16& L, uint32_t g, uint32_t& w01, uint32_t& w23) {
  const uint32_t s = g & 0x7777u;                        // entry index within a group of 8
  const uint32_t sel = ((g >> 1) & 0x4444u) | 0x3210u;   // take the upper group where bit 3 is set
  const uint32_t lo = __byte_perm(__byte_perm(L.lo[0], L.lo[1], s), __byte_perm(L.lo[2], L.lo[3], s), sel);
  const uint32_t hi = __byte_perm(__byte_perm(L.hi[0], L.hi[1], s), __byte_perm(L.hi[2], L.hi[3], s), sel);
  // nibble order of g is element 1, 0, 3, 2
  w01 = __byte_perm(lo, hi, 0x4051);
  w23 = __byte_perm(lo, hi, 0x6273);
}

// 8 codes (one 32-bit word) -> 8 bf16 (one 16-byte chunk).
__device__ __forceinline__ uint4 lut_lookup8(const Lut16& L, uint32_t w) {
  uint4 o;
  lut_lookup4(L, w, o.x, o.y);
  lut_lookup4(L, w >> 16, o.z, o.w);
  return o;
}

// ====================================================================== code-byte pair table
//
// A 64 KB shared-memory table that turns one packed code byte (element 2k in
// the high nibble, element 2k+1 in the low nibble) into its two fp32 code
// values with a single 8-byte load.  For byte value v and replica r (0..15)
// the pair {q[v >> 4], q[v & 15]} sits at  T + 256 v + 8 r.  A lane reads
// replica (lane & 15): the 16 lanes of each half-warp then cover the 32 banks
// exactly once, whatever the bytes, so every lookup is conflict-free (two
// shared-memory wavefronts per warp, the minimum for 8-byte loads).  T is a
// multiple of 65536 in the shared window, so one byte permute assembles the
// whole address from the code byte and a per-lane key {8 r, -, T >> 16, 0}.
constexpr uint32_t kPairTabBytes = 65536;

__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

// Offset, from the start of dynamic shared memory, of the first 64 KB-aligned
// window address at least min_offset bytes in; the caller checks
// offset + kPairTabBytes (+ whatever follows) <= its size.
__device__ __forceinline__ uint32_t pair_tab_offset(const void* dsmem, uint32_t min_offset = 0) {
  const uint32_t base = smem_u32(dsmem);
  return ((base + min_offset + 0xFFFFu) & ~0xFFFFu) - base;
}

// Fills the table at tab (whose window address is a multiple of 65536) from
// the 16 code values q; every thread of the block takes part.
__device__ __forceinline__ void fill_pair_table(uint8_t* tab, const float* q) {
  for (int i = threadIdx.x; i < 256 * 16; i += blockDim.x) {
    const int v = i >> 4, r = i & 15;
    *reinterpret_cast<float2*>(tab + v * 256 + r * 8) = make_float2(q[v >> 4], q[v & 15]);
  }
}

__device__ __forceinline__ uint32_t pair_key(const uint8_t* tab, int lane) {
  return smem_u32(tab) | (static_cast<uint32_t>(lane & 15) * 8u);
}

// {c, c} as one 64-bit operand of the paired multiply.
__device__ __forceinline__ uint64_t dup_f32x2(float c) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(c));
  return r;
}

// Byte J of the code word w -> the fp32 pair {q[hi], q[lo]} (the element of the
// high nibble in the low word): one byte permute (address) and one 8-byte
// shared load.
template <int J>
__device__ __forceinline__ uint64_t pair_values(uint32_t w, uint32_t key) {
  const uint32_t addr = __byte_perm(w, key, 0x7604u | (J << 4));
  uint64_t qq;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(qq) : "r"(addr));
  return qq;
}

// Byte J of the code word w -> bf16x2 {bf16(q[hi] * c), bf16(q[lo] * c)}, the
// element of the high nibble in the low half: the pair lookup, one paired fp32
// multiply (IEEE round-to-nearest per lane, identical to two separate
// multiplies) and one paired conversion.
template <int J>
__device__ __forceinline__ uint32_t pair_dequant(uint32_t w, uint32_t key, uint64_t cc) {
  const uint64_t qq = pair_values<J>(w, key);
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(qq), "l"(cc));
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
  return pack_bf16x2(a, b);
}

// 8 codes (one 32-bit word) -> 8 bf16 in element order (16 bytes).
__device__ __forceinline__ uint4 word_dequant(uint32_t w, uint32_t key, uint64_t cc) {
  return make_uint4(pair_dequant<0>(w, key, cc), pair_dequant<1>(w, key, cc), pair_dequant<2>(w, key, cc),
                    pair_dequant<3>(w, key, cc));
}

// Block constant c' with the per-group division cached: dq_scale / 448 is
// recomputed only when the group's scale changes.
struct ConstCache {
  uint32_t scale_bits = 0xFFFFFFFFu;
  float step = 0.0f;
  __device__ __forceinline__ float constant(uint8_t e, float scale, float mu) {
    if (__float_as_uint(scale) != scale_bits) {
      scale_bits = __float_as_uint(scale);
      step = __fdiv_rn(scale, 448.0f);
    }
    return __fadd_rn(__fmul_rn(e4m3_to_float(e), step), mu);
  }
};

// ------------------------------------------------------------------ LoRA dropout draws

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): each round multiplies words 0 and 2
// of the counter by two 32-bit constants into 64-bit products and forms the
// next counter from their halves, the other two words and the key; the key
// advances by two Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    if (rnd) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = c.x * 0xD2511F53u, hi0 = __umulhi(c.x, 0xD2511F53u);
    const uint32_t lo1 = c.z * 0xCD9E8D57u, hi1 = __umulhi(c.z, 0xCD9E8D57u);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// Keep bits of the adapter-input elements 4b .. 4b + 3 (flat index of X):
// element 4b + j is kept when word j of Philox at counter (b, 0, 0) under the
// key `seed` is at least thr = floor(p 2^32).  Bit j of the result.
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t b, uint64_t seed, uint32_t thr) {
  const uint4 r = philox4x32_10(make_uint4(static_cast<uint32_t>(b), static_cast<uint32_t>(b >> 32), 0u, 0u),
                                static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  return (r.x >= thr ? 1u : 0u) | (r.y >= thr ? 2u : 0u) | (r.z >= thr ? 4u : 0u) | (r.w >= thr ? 8u : 0u);
}

// Zeroes the bf16 halves of the pair w whose keep bit (bits 0 and 1 of k) is clear.
__device__ __forceinline__ uint32_t keep_pair(uint32_t w, uint32_t k) {
  return w & ((k & 1u ? 0x0000FFFFu : 0u) | (k & 2u ? 0xFFFF0000u : 0u));
}

// Programmatic dependent launch.// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel before it in the stream is still
// running, once every CTA of that kernel has executed launch_dependents (or
// exited); pdl_wait blocks until that kernel has completed and its memory is
// visible (it returns at once when the launch did not use the attribute).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// FP8 constants and second-level scales for a thread that walks one weight
// row a few blocks at a time.  The constants are read as aligned 16-byte
// chunks of the flat block array (one load serves 16 blocks instead of one
// byte gather per block, the chunk after it prefetched into L1) and the scale
// is re-read only when the 256-block group changes.  nblk bounds the array:
// the last partial chunk, and an array that is not 16-byte aligned, are read
// byte by byte.
struct ConstWindow {
  int64_t chunk = -1;
  uint4 bytes = make_uint4(0u, 0u, 0u, 0u);
  int64_t group = -1;
  float scale = 0.0f;
  __device__ __forceinline__ void get(const uint8_t* __restrict__ absmax, const float* __restrict__ dq_scale,
                                      int64_t nblk, int64_t blk, uint32_t& e8, float& s32) {
    const int64_t c = blk >> 4;
    if (c != chunk) {
      chunk = c;
      const int64_t b0 = c << 4;
      if (b0 + 16 <= nblk && (reinterpret_cast<uintptr_t>(absmax) & 15u) == 0) {
        bytes = __ldg(reinterpret_cast<const uint4*>(absmax + b0));
        if (b0 + 32 <= nblk) asm volatile("prefetch.global.L1 [%0];" ::"l"(absmax + b0 + 16));
      } else {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (b0 + i < nblk) w[i >> 2] |= static_cast<uint32_t>(__ldg(absmax + b0 + i)) << (8 * (i & 3));
        bytes = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    const int b = static_cast<int>(blk & 15);
    const uint32_t word = b < 8 ? (b < 4 ? bytes.x : bytes.y) : (b < 12 ? bytes.z : bytes.w);
    e8 = (word >> (8 * (b & 3))) & 0xFFu;
    const int64_t g = blk >> 8;
    if (g != group) {
      group = g;
      scale = __ldg(dq_scale + g);
    }
    s32 = scale;
  }
};

}  // namespace qlora
