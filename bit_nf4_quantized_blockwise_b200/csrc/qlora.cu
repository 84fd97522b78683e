// qlora.cu - the C ABI of libqlora.so (declared in include/qlora.h).
//
// One translation unit: argument validation, tensor-map construction and
// kernel launches for NF4 quantization, double quantization, dequantization
// and the QLoRA linear layer forward / backward.  Every entry point validates
// its arguments before it enqueues anything and never synchronizes the host
// (except qlora_check_status, whose job is to wait).
#include "qlora.h"

#include "common.cuh"
#include "gemm.cuh"
#include "optim.cuh"
#include "pairgemm.cuh"
#include "quant.cuh"

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

using namespace qlora;

namespace {

constexpr int kVersion = 10000;  // 1.0.0
// Forward calls with at most kSmallMMax tokens take a small-M (decode) kernel:
// the register-fed MMA kernel up to kDecodeMMax tokens (one or two 8-token
// MMA column groups), the tcgen05 kernel with the weight in tensor memory
// above that.
constexpr int64_t kSmallMMax = 32;
constexpr int64_t kDecodeMMax = SD_MAX_TOKENS;

// ------------------------------------------------------------------ launch counting and tracing
//
// Every kernel launch increments a counter.  With tracing on, each launch is
// bracketed by two CUDA events recorded on its own stream, so that a caller
// can read the device time of each kernel family afterwards.

std::atomic<long long> g_launches{0};

struct TraceRec {
  int family;
  cudaEvent_t start, stop;
};

struct Tracer {
  std::mutex mu;
  bool on = false;
  std::vector<TraceRec> recs;
  std::vector<cudaEvent_t> pool;

  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

Tracer& tracer() {
  static Tracer t;
  return t;
}

// Brackets one kernel launch: counts it and, with tracing on, records events.
class LaunchScope {
 public:
  LaunchScope(int family, cudaStream_t st) : family_(family), st_(st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    Tracer& t = tracer();
    std::lock_guard<std::mutex> lock(t.mu);
    if (!t.on) return;
    start_ = t.get();
    stop_ = t.get();
    if (start_ && stop_) cudaEventRecord(start_, st_);
  }
  ~LaunchScope() {
    if (!start_ || !stop_) return;
    cudaEventRecord(stop_, st_);
    Tracer& t = tracer();
    std::lock_guard<std::mutex> lock(t.mu);
    t.recs.push_back({family_, start_, stop_});
  }

 private:
  int family_;
  cudaStream_t st_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_codebook(const float* q) {
  int zeros = 0;
  for (int j = 0; j < 16; ++j) {
    if (!std::isfinite(q[j])) return QLORA_ERR_CODEBOOK;
    if (q[j] == 0.0f) ++zeros;
    if (j > 0 && !(q[j] > q[j - 1])) return QLORA_ERR_CODEBOOK;
  }
  return zeros == 1 ? QLORA_OK : QLORA_ERR_CODEBOOK;
}

int zero_index(const float* q) {
  for (int j = 0; j < 16; ++j)
    if (q[j] == 0.0f) return j;
  return -1;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int64_t grid_for(int64_t work_items, int per_cta, int max_ctas) {
  int64_t g = (work_items + per_cta - 1) / per_cta;
  if (g > max_ctas) g = max_ctas;
  return g < 1 ? 1 : g;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ------------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [outer][inner] array with the given row pitch.
bool map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D uint8 map over a row-major [outer][inner] byte array (no swizzle unless
// asked; an N-byte swizzle needs box_inner == N).
bool map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
            uint32_t box_outer, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map, dims {d0, d1, d2} (innermost first) with byte strides s1, s2
// of dims 1 and 2, box {b0, b1, b2}, 128-byte swizzle (b0 * 2 must be 128).
bool map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                 uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ quantizer decision table cache

struct TableCache {
  std::mutex mu;
  bool valid = false;
  float q[16];
  BoundaryTable table;
};

TableCache& table_cache() {
  static TableCache c;
  return c;
}

bool get_table(const float* q, BoundaryTable* out) {
  TableCache& c = table_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  if (!c.valid || std::memcmp(c.q, q, sizeof(c.q)) != 0) {
    float t[15];
    nf4_thresholds(q, t);
    if (!build_boundary_table(t, &c.table)) return false;
    std::memcpy(c.q, q, sizeof(c.q));
    c.valid = true;
  }
  *out = c.table;
  return true;
}

// ------------------------------------------------------------------ kernel attributes

template <typename K>
int set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

int check_wq(const qlora_nf4_t* Wq) {
  if (!Wq) return QLORA_ERR_NULL;
  if (!Wq->codes) return QLORA_ERR_NULL;
  if (Wq->block != QLORA_BLOCK) return QLORA_ERR_UNSUPPORTED;
  if (Wq->o <= 0 || Wq->h <= 0 || Wq->h % 64 != 0) return QLORA_ERR_SHAPE;
  if (!aligned16(Wq->codes)) return QLORA_ERR_ALIGN;
  if (Wq->absmax) {
    // single-level constants: one fp32 per block
    if (!aligned16(Wq->absmax)) return QLORA_ERR_ALIGN;
  } else {
    if (!Wq->absmax_fp8 || !Wq->dq_scale || !Wq->dq_mean) return QLORA_ERR_NULL;
    if (Wq->dq_block != QLORA_DQ_BLOCK) return QLORA_ERR_UNSUPPORTED;
    if ((Wq->o * Wq->h) % (64 * 256) != 0) return QLORA_ERR_SHAPE;
    if (!aligned16(Wq->absmax_fp8) || !aligned16(Wq->dq_scale)) return QLORA_ERR_ALIGN;
  }
  return check_codebook(Wq->codebook);
}

// T-style rank-r GEMM launch:  D (+)= A * (B [+ B2]).
// Dropout of the adapter input: keep threshold floor(p 2^32) (0: no dropout),
// the Philox key and the fp32 scale 1 / (1 - p).
struct DropoutCfg {
  uint32_t thr = 0;
  uint64_t seed = 0;
  float scale = 1.0f;
  bool on() const { return thr != 0; }
};

// T-style rank-r GEMM launch:  D (+)= alpha * A * (B [+ B2]), optionally times
// the dropout keep bit of element (m, n) of a row-major [rows][mask_ld] array.
template <bool kAmn, bool kBmn>
int launch_tgemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, int rows, int cols,
                 int k_elems, bool hilo, float* out, int64_t ld, bool transpose, cudaStream_t st,
                 float alpha = 1.0f, const DropoutCfg* mask = nullptr, int64_t mask_ld = 0) {
  TGemmParams p{};
  p.M = rows;
  p.N = cols;
  p.bn = ((cols + 63) / 64) * 64;
  if (p.bn > 256) p.bn = 256;
  p.alpha = alpha;
  if (mask) {
    p.mask_thr = mask->thr;
    p.mask_seed = mask->seed;
    p.mask_ld = mask_ld;
  }
  p.k_stages = (k_elems + TG_BK - 1) / TG_BK;
  p.hilo = hilo ? 1 : 0;
  const int stage_bytes = TG_BM * TG_BK * 2 + (hilo ? 2 : 1) * p.bn * TG_BK * 2;
  // a ring of at least two stages; two CTAs per SM when two such rings fit
  int per_sm = 2;
  p.stages = TG_SMEM_LIMIT / stage_bytes;
  if (p.stages < 2) {
    per_sm = 1;
    p.stages = TG_SMEM_LIMIT_ONE / stage_bytes;
  }
  if (p.stages > TG_MAX_STAGES) p.stages = TG_MAX_STAGES;
  if (p.stages < 2) return QLORA_ERR_UNSUPPORTED;
  const int tiles = ((rows + TG_BM - 1) / TG_BM) * ((cols + p.bn - 1) / p.bn);
  const int sms = sm_count();
  // split the reduction so that all CTAs fit one wave (a second, nearly empty
  // wave would double the time of these short kernels)
  int splits = (per_sm * sms) / tiles;
  if (splits > p.k_stages) splits = p.k_stages;
  if (splits < 1) splits = 1;
  p.k_per_split = (p.k_stages + splits - 1) / splits;
  splits = (p.k_stages + p.k_per_split - 1) / p.k_per_split;
  p.out = out;
  p.ld_out = ld;
  p.transpose_out = transpose ? 1 : 0;
  const int smem = p.stages * stage_bytes + 1024 + 256;
  if (set_smem(gemm_tma_kernel<kAmn, kBmn>, smem) != QLORA_OK) return QLORA_ERR_CUDA;
  dim3 grid((rows + TG_BM - 1) / TG_BM, (cols + p.bn - 1) / p.bn, splits);
  {
    LaunchScope ls(QLORA_KERNEL_TGEMM, st);
    gemm_tma_kernel<kAmn, kBmn><<<grid, TG_THREADS, smem, st>>>(a, b, b2, p);
  }
  return launch_status();
}

// Workspace layout shared by the forward and backward passes.
struct LoraWs {
  float* U;        // [M][r] fp32 (backward only)
  uint16_t* UU;    // [M][KL] bf16 hi|lo (backward only)
  float* T;        // [M][r] fp32
  uint16_t* TT;    // [M][KL] bf16 hi|lo
  uint16_t* L1x;   // [h][KL] = [L1 | 0 | L1 | 0]
  uint16_t* L2x;   // [o][KL] = [L2^T | 0 | L2^T | 0]
  float* Yacc;     // [M][o] fp32 accumulator of the small-M forward (bf16 output only)
  float* P;        // [n_part][M][r] fp32 partials of X L1 (register-fed MMA decode forward)
  uint16_t* Xm;    // [M][h] bf16, the adapter input after dropout (dropout calls)
  float* dXf;      // [M][h] fp32 accumulator of dX (dropout backward)
  uint16_t* Wd;    // [o][h] bf16, the dequantized weight W'^T (calls of kPairMMin tokens or more)
  float* Wpart;    // [pairs][256][256] fp32 partial accumulators of the pair-tile GEMM's split tiles
  unsigned* Wcnt;  // [pairs][8] arrival counters of the split tiles
  size_t bytes;
};

// Calls of at least this many tokens dequantize W' once into the workspace and
// run the pair-tile bf16 GEMM; below it the fused dequant-GEMM expands W' per
// 256-row tile (when the workspace cannot hold W', the fused kernel runs too).
constexpr int64_t kPairMMin = 1024;

LoraWs lora_ws_layout(void* base, int64_t o, int64_t h, int64_t M, int r, bool bwd, bool dropout = false,
                      bool wprime = false) {
  const int64_t rp = ((r + 63) / 64) * 64;
  const int64_t KL = 2 * rp;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  LoraWs w{};
  auto take = [&](size_t bytes) -> void* {
    void* q = p ? p + off : nullptr;
    off += round256(bytes);
    return q;
  };
  // Forward calls of up to kSmallMMax tokens (decode) compute T without packed
  // L1; those of up to kDecodeMMax tokens (register-fed MMA kernel) keep T as
  // per-CTA partials and need neither the split T nor packed L2.
  const bool fwd_small = !bwd && M <= kSmallMMax, fwd_dec = !bwd && M <= kDecodeMMax;
  if (bwd) {
    w.U = static_cast<float*>(take(static_cast<size_t>(M) * r * 4));
    w.UU = static_cast<uint16_t*>(take(static_cast<size_t>(M) * KL * 2));
  }
  if (!fwd_dec) {
    w.T = static_cast<float*>(take(static_cast<size_t>(M) * r * 4));
    w.TT = static_cast<uint16_t*>(take(static_cast<size_t>(M) * KL * 2));
    w.L2x = static_cast<uint16_t*>(take(static_cast<size_t>(o) * KL * 2));
  }
  if (!fwd_small) w.L1x = static_cast<uint16_t*>(take(static_cast<size_t>(h) * KL * 2));
  if (fwd_small) w.Yacc = static_cast<float*>(take(static_cast<size_t>(M) * o * 4));
  if (fwd_dec) {
    const int64_t n_part = (h + rank_r_rows(r) - 1) / rank_r_rows(r);
    w.P = static_cast<float*>(take(static_cast<size_t>(n_part) * M * r * 4));
  }
  // with dropout, the masked adapter input feeds the tensor-core products of
  // T and dL1 (decode forwards mask it inside the rank-r kernel instead), and
  // the backward accumulates dX in fp32 before a bf16 output is written
  if (dropout && !fwd_small) w.Xm = static_cast<uint16_t*>(take(static_cast<size_t>(M) * h * 2));
  if (dropout && bwd) w.dXf = static_cast<float*>(take(static_cast<size_t>(M) * h * 4));
  if (wprime && M >= kPairMMin) {
    const size_t pairs = static_cast<size_t>((sm_count() + 1) / 2);
    w.Wd = static_cast<uint16_t*>(take(static_cast<size_t>(o) * h * 2));
    w.Wpart = static_cast<float*>(take(pairs * PG_BM * PG_BN * 4));
    w.Wcnt = static_cast<unsigned*>(take(pairs * 8 * 4));
  }
  w.bytes = off;
  return w;
}

// Dequantizes the whole weight to bf16 W'^T [o][h] (the same kernel as qlora_dequant).
int dequant_into(const qlora_nf4_t* Wq, uint16_t* out, int family, cudaStream_t st) {
  DequantParams p{};
  p.codes = reinterpret_cast<const uint32_t*>(Wq->codes);
  p.absmax_fp8 = Wq->absmax_fp8;
  p.dq_scale = Wq->dq_scale;
  p.dq_mean = Wq->dq_mean;
  p.absmax32 = Wq->absmax;
  p.out = reinterpret_cast<uint4*>(out);
  p.nwords = Wq->o * Wq->h / 8;
  p.nblocks = Wq->o * Wq->h / 64;
  std::memcpy(p.codebook, Wq->codebook, sizeof(p.codebook));
  if (set_smem(nf4_dequant_kernel, kDequantSmem) != QLORA_OK) return QLORA_ERR_CUDA;
  const int64_t grid = grid_for(p.nwords, kDequantThreads * kDequantWords, sm_count());
  {
    LaunchScope ls(family, st);
    nf4_dequant_kernel<<<static_cast<unsigned>(grid), kDequantThreads, kDequantSmem, st>>>(p);
  }
  return launch_status();
}

// Two-CTA clusters of the pair-tile GEMM that can be resident at once (one per
// SM pair when nothing else runs), per device.
template <bool kBwd>
int resident_pairs() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cache[dev].load();
  if (n > 0) return n;
  if (set_smem(pair_gemm_kernel<kBwd>, PG_SMEM_BYTES) != QLORA_OK) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * static_cast<unsigned>((sm_count() + 1) / 2), 1, 1);
  cfg.blockDim = dim3(PG_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PG_SMEM_BYTES;
  if (cudaOccupancyMaxActiveClusters(&n, pair_gemm_kernel<kBwd>, &cfg) != cudaSuccess || n <= 0) return 0;
  cache[dev].store(n);
  return n;
}

// D = A (op W') + A_ext B_ext with W'^T [o][h] dequantized in memory: tokens
// M, output columns N, reduction K over W' (forward: N = o, K = h; backward:
// N = h, K = o), LoRA extension KL (0: none).  Persistent: as many two-CTA
// clusters as can be resident, tiles ordered N-fastest.
template <bool kBwd>
int launch_pair_gemm(const void* A, int64_t M, int64_t K, const uint16_t* Wd, int64_t o, int64_t h,
                     const uint16_t* Ae, const uint16_t* Be, int64_t KL, void* out, int out_bf16, const LoraWs& w,
                     int family, cudaStream_t st) {
  const int64_t N = kBwd ? h : o;
  CUtensorMap ma, mb, mae, mbe;
  if (!map_bf16(&ma, A, K, M, K * 2, 64, 128)) return QLORA_ERR_CUDA;
  if (!map_bf16(&mb, Wd, h, o, h * 2, 64, 128)) return QLORA_ERR_CUDA;
  if (KL > 0) {
    if (!map_bf16(&mae, Ae, KL, M, KL * 2, 64, 128)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mbe, Be, KL, N, KL * 2, 64, 128)) return QLORA_ERR_CUDA;
  } else {
    mae = ma;
    mbe = mb;
  }
  PairGemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.k_main_stages = static_cast<int>((K + PG_BK - 1) / PG_BK);
  p.k_ext_stages = static_cast<int>(KL / PG_BK);
  p.n_tiles = static_cast<int>((N + PG_BN - 1) / PG_BN);
  p.units = static_cast<int>((M + PG_BM - 1) / PG_BM) * p.n_tiles;
  p.out = out;
  p.out_bf16 = out_bf16;
  p.ld_out = N;
  int pairs = resident_pairs<kBwd>();
  if (pairs <= 0) return QLORA_ERR_CUDA;
  if (pairs > (sm_count() + 1) / 2) pairs = (sm_count() + 1) / 2;  // the partial buffer's bound
  if (set_smem(pair_gemm_kernel<kBwd>, PG_SMEM_BYTES) != QLORA_OK) return QLORA_ERR_CUDA;
  const int clusters = p.units < pairs ? p.units : pairs;
  // A last round with fewer tiles than pairs is split along K into up to four
  // parts per tile (each at least two stages), so that it lasts a part.
  const int tail = p.units % clusters;
  const int S = p.k_main_stages + p.k_ext_stages;
  int split = tail > 0 ? clusters / tail : 1;
  if (split > 4) split = 4;
  if (split > S / 2) split = S / 2;
  if (split < 2) split = 1;
  p.split = split;
  p.full_units = split > 1 ? p.units - tail : p.units;
  p.partial = w.Wpart;
  p.counters = w.Wcnt;
  if (split > 1 && cudaMemsetAsync(w.Wcnt, 0, static_cast<size_t>(tail) * 8 * 4, st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  {
    LaunchScope ls(family, st);
    pair_gemm_kernel<kBwd><<<2 * clusters, PG_THREADS, PG_SMEM_BYTES, st>>>(ma, mb, mae, mbe, p);
  }
  return launch_status();
}

int check_linear_args(const qlora_nf4_t* Wq, int64_t M, int r, int dtype) {
  const int s = check_wq(Wq);
  if (s != QLORA_OK) return s;
  if (r < 8 || r > QLORA_MAX_RANK || r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (dtype != QLORA_DTYPE_F32 && dtype != QLORA_DTYPE_BF16) return QLORA_ERR_UNSUPPORTED;
  if (M < 1 || M > (int64_t(1) << 31) - 1) return QLORA_ERR_SHAPE;
  if (Wq->o % 64 != 0 || Wq->o > (int64_t(1) << 30) || Wq->h > (int64_t(1) << 30)) return QLORA_ERR_SHAPE;
  return QLORA_OK;
}

// Common front half, two launches: one packing kernel (L1x, L2x and the
// zeroing of every fp32 accumulator of the call) and, unless T is given, the
// rank-r GEMM T = X L1.
struct ZeroList {
  float* ptr[3] = {nullptr, nullptr, nullptr};
  int64_t len[3] = {0, 0, 0};
};

// Packs the LoRA factors for the tensor-core kernels, zeroes the listed
// accumulators and computes T = X L1.  small: T for a decode call (M <= 32)
// by the split-K rank-r kernel on CUDA cores (no L1 packing); otherwise by the
// tensor-core GEMM on packed L1.
int lora_prep(const qlora_nf4_t* Wq, const void* X, int64_t M, const void* L1, const void* L2, int r,
              const LoraWs& w, float* T, bool compute_T, const ZeroList& zeros, cudaStream_t st,
              bool small = false, const DropoutCfg& d = DropoutCfg()) {
  const int64_t o = Wq->o, h = Wq->h;
  const int rp = ((r + 63) / 64) * 64;
  const int KL = 2 * rp;
  PrepParams pp{};
  pp.L1 = static_cast<const uint16_t*>(L1);
  pp.L2 = static_cast<const uint16_t*>(L2);
  pp.L1x = small ? nullptr : w.L1x;
  pp.L2x = w.L2x;
  pp.h = h;
  pp.o = o;
  pp.r = r;
  pp.rp = rp;
  int nz = 0;
  if (compute_T) {
    pp.zero_ptr[nz] = T;
    pp.zero_len[nz++] = M * r;
  }
  for (int i = 0; i < 3; ++i)
    if (zeros.ptr[i]) {
      pp.zero_ptr[nz] = zeros.ptr[i];
      pp.zero_len[nz++] = zeros.len[i];
    }
  const int64_t rows = (o > h ? o : h);
  int64_t gx = (rows + 31) / 32;
  if (!pp.L1x && !pp.L2x && gx > 2 * sm_count()) gx = 2 * sm_count();  // only the zeroing job has work
  dim3 grid(static_cast<unsigned>(gx), 3);
  {
    LaunchScope ls(QLORA_KERNEL_AUX, st);
    lora_prep_kernel<<<grid, 256, 0, st>>>(pp);
  }
  if (launch_status() != QLORA_OK) return QLORA_ERR_CUDA;
  if (small) {
    {
      LaunchScope ls(QLORA_KERNEL_TGEMM, st);
      const int rows = rank_r_rows(r);
      rank_r_small_kernel<<<static_cast<unsigned>((h + rows - 1) / rows), 256, 0, st>>>(
          static_cast<const uint16_t*>(X), static_cast<int>(M), h, static_cast<const uint16_t*>(L1), r,
          compute_T ? T : nullptr, nullptr, nullptr, 0, d.thr, d.seed, d.scale);
    }
    return launch_status();
  }
  if (compute_T) {
    // with dropout the adapter input is the masked copy, and T takes the scale
    const void* XT = d.on() ? static_cast<const void*>(w.Xm) : X;
    if (d.on()) {
      LaunchScope ls(QLORA_KERNEL_AUX, st);
      const int64_t nvec = M * h / 8;
      dropout_mask_kernel<<<static_cast<unsigned>(grid_for(nvec, 256, sm_count() * 8)), 256, 0, st>>>(
          static_cast<const uint4*>(X), nvec, reinterpret_cast<uint4*>(w.Xm), d.thr, d.seed);
    }
    CUtensorMap ma, mb;
    // T = X L1: A = X K-major [M][h]; B(n=j, k=i) = L1x[i][j], MN-major.
    if (!map_bf16(&ma, XT, h, M, h * 2, 64, 128)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb, w.L1x, rp, h, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    const int rc = launch_tgemm<false, true>(ma, mb, mb, static_cast<int>(M), r, static_cast<int>(h), false, T, r,
                                             false, st, d.scale);
    if (rc != QLORA_OK) return rc;
  }
  return QLORA_OK;
}

// hi/lo split of s * src into dst for one or two (src, dst) pairs, one launch.
int lora_split(const float* src0, uint16_t* dst0, const float* src1, uint16_t* dst1, int64_t M, int r, float s,
               cudaStream_t st) {
  const int rp = ((r + 63) / 64) * 64;
  const int KL = 2 * rp;
  SplitJob j0{src0, dst0}, j1{src1, dst1};
  dim3 grid(static_cast<unsigned>(grid_for(M * KL, 256, sm_count() * 4)), src1 ? 2 : 1);
  {
    LaunchScope ls(QLORA_KERNEL_AUX, st);
    lora_split_kernel<<<grid, 256, 0, st>>>(j0, j1, M, r, rp, s);
  }
  return launch_status();
}

// Failure-path probe: one thread waits on an mbarrier that nothing arrives on,
// with a short limit, so the wait gives up the way a stalled pipeline would.
// No copy and no MMA is in flight; the kernel returns after the limit.
__global__ void wait_probe_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, kTagWaitProbe, limit_ns);
}

}  // namespace

// ====================================================================== public entry points

extern "C" {

const char* qlora_status_string(int status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "null pointer";
    case QLORA_ERR_SHAPE: return "invalid shape";
    case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLORA_ERR_UNSUPPORTED: return "unsupported parameter";
    case QLORA_ERR_CODEBOOK: return "invalid codebook";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "kernel pipeline wait timed out";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_SCRATCH_LIMIT: return "problem needs more than the no-allocation call's built-in scratch";
    default: return "unknown status";
  }
}

int qlora_version(void) { return kVersion; }

int qlora_nf4_codebook(float* out) {
  if (!out) return QLORA_ERR_NULL;
  nf4_code_values(out);
  return check_codebook(out);
}

int qlora_nf4_boundaries(const float* codebook, uint16_t* out) {
  if (!codebook || !out) return QLORA_ERR_NULL;
  const int cb = check_codebook(codebook);
  if (cb != QLORA_OK) return cb;
  float t[15];
  nf4_thresholds(codebook, t);
  BoundaryTable tab;
  if (!build_boundary_table(t, &tab)) return QLORA_ERR_CODEBOOK;
  std::memcpy(out, tab.b, sizeof(tab.b));
  return QLORA_OK;
}

int qlora_quantize_nf4(const void* W, int64_t n, const float* codebook, int block, uint8_t* codes, float* absmax,
                       void* stream) {
  if (!W || !codebook || !codes || !absmax) return QLORA_ERR_NULL;
  if (block != QLORA_BLOCK) return QLORA_ERR_UNSUPPORTED;
  if (n <= 0 || n % 64 != 0) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(absmax)) return QLORA_ERR_ALIGN;
  const int cb = check_codebook(codebook);
  if (cb != QLORA_OK) return cb;
  QuantizeParams p{};
  BoundaryTable tab;
  if (!get_table(codebook, &tab)) return QLORA_ERR_CODEBOOK;
  nf4_thresholds(codebook, p.t);
  p.t[15] = 0.0f;
  p.zero_code = static_cast<uint32_t>(zero_index(codebook));
  p.fast_ok = tab.ok ? 1u : 0u;
  p.bin_ok = tab.ok && tab.bins_ok ? 1u : 0u;
  for (int m = 0; m < 128; ++m)
    for (int j = 0; j < 16; ++j) p.bnd[m][j] = static_cast<uint32_t>(tab.b[m][j]) * 0x00010001u;
  p.w = static_cast<const uint4*>(W);
  p.codes = reinterpret_cast<uint2*>(codes);
  p.absmax = absmax;
  p.nblocks = n / 64;
  // with the bin table (64 KB of shared memory per CTA) three CTAs fit an SM
  const int smem = p.bin_ok ? kQuantBinSmem : 0;
  if (smem && set_smem(nf4_quantize_kernel, smem) != QLORA_OK) return QLORA_ERR_CUDA;
  const int64_t grid = grid_for(p.nblocks, 128, sm_count() * (p.bin_ok ? 3 : 4));
  {
    LaunchScope ls(QLORA_KERNEL_QUANTIZE, static_cast<cudaStream_t>(stream));
    nf4_quantize_kernel<<<static_cast<unsigned>(grid), 256, smem, static_cast<cudaStream_t>(stream)>>>(p);
  }
  return launch_status();
}

size_t qlora_double_quant_workspace_size(int64_t nblocks, int dq_block) {
  (void)nblocks;
  (void)dq_block;
  return 256;
}

int qlora_double_quant(const float* absmax, int64_t nblocks, int dq_block, uint8_t* absmax_fp8, float* dq_scale,
                       float* dq_mean, void* ws, size_t ws_bytes, void* stream) {
  if (!absmax || !absmax_fp8 || !dq_scale || !dq_mean) return QLORA_ERR_NULL;
  if (dq_block != QLORA_DQ_BLOCK) return QLORA_ERR_UNSUPPORTED;
  if (nblocks <= 0 || nblocks % QLORA_DQ_BLOCK != 0) return QLORA_ERR_SHAPE;
  if (!ws || ws_bytes < qlora_double_quant_workspace_size(nblocks, dq_block)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(absmax) || !aligned16(absmax_fp8) || !aligned16(ws)) return QLORA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* sum = static_cast<double*>(ws);
  if (cudaMemsetAsync(sum, 0, sizeof(double), st) != cudaSuccess) return QLORA_ERR_CUDA;
  const int sms = sm_count();
  const int64_t n4 = nblocks / 4;
  {
    LaunchScope ls(QLORA_KERNEL_DOUBLE_QUANT, st);
    dq_sum_kernel<<<static_cast<unsigned>(grid_for(n4, 1024, sms)), 256, 0, st>>>(
        reinterpret_cast<const float4*>(absmax), n4, sum);
  }
  const int64_t ngroups = nblocks / QLORA_DQ_BLOCK;
  {
    LaunchScope ls(QLORA_KERNEL_DOUBLE_QUANT, st);
    dq_encode_kernel<<<static_cast<unsigned>(grid_for(ngroups, 8, sms * 8)), 256, 0, st>>>(
        reinterpret_cast<const float4*>(absmax), ngroups, nblocks, sum, reinterpret_cast<uint2*>(absmax_fp8),
        dq_scale, dq_mean);
  }
  return launch_status();
}

int qlora_dequant(const qlora_nf4_t* Wq, void* out, void* stream) {
  const int s = check_wq(Wq);
  if (s != QLORA_OK) return s;
  if (!out) return QLORA_ERR_NULL;
  if (!aligned16(out)) return QLORA_ERR_ALIGN;
  DequantParams p{};
  p.codes = reinterpret_cast<const uint32_t*>(Wq->codes);
  p.absmax_fp8 = Wq->absmax_fp8;
  p.dq_scale = Wq->dq_scale;
  p.dq_mean = Wq->dq_mean;
  p.absmax32 = Wq->absmax;
  p.out = static_cast<uint4*>(out);
  p.nwords = Wq->o * Wq->h / 8;
  p.nblocks = Wq->o * Wq->h / 64;
  std::memcpy(p.codebook, Wq->codebook, sizeof(p.codebook));
  if (set_smem(nf4_dequant_kernel, kDequantSmem) != QLORA_OK) return QLORA_ERR_CUDA;
  const int64_t grid = grid_for(p.nwords, kDequantThreads * kDequantWords, sm_count());
  {
    LaunchScope ls(QLORA_KERNEL_DEQUANT, static_cast<cudaStream_t>(stream));
    nf4_dequant_kernel<<<static_cast<unsigned>(grid), kDequantThreads, kDequantSmem,
                         static_cast<cudaStream_t>(stream)>>>(p);
  }
  return launch_status();
}

size_t qlora_linear_fwd_workspace_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, false, false, true).bytes;
}

size_t qlora_linear_bwd_workspace_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, true, false, true).bytes;
}

size_t qlora_linear_fwd_workspace_min_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, false).bytes;
}

size_t qlora_linear_bwd_workspace_min_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, true).bytes;
}

}  // extern "C"

namespace {

int linear_fwd_impl(const qlora_nf4_t* Wq, const void* X, int64_t M, const void* L1, const void* L2, int r, float s,
                    const DropoutCfg& d, void* Y, int y_dtype, float* T_save, void* ws, size_t ws_bytes,
                    void* stream) {
  int rc = check_linear_args(Wq, M, r, y_dtype);
  if (rc != QLORA_OK) return rc;
  if (!X || !L1 || !L2 || !Y) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(L1) || !aligned16(L2) || !aligned16(Y) || (T_save && !aligned16(T_save)) ||
      (ws && !aligned16(ws)))
    return QLORA_ERR_ALIGN;
  const int64_t o = Wq->o, h = Wq->h;
  if (!ws || ws_bytes < lora_ws_layout(nullptr, o, h, M, r, false, d.on()).bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pair = M >= kPairMMin && ws_bytes >= lora_ws_layout(nullptr, o, h, M, r, false, d.on(), true).bytes;
  const LoraWs w = lora_ws_layout(ws, o, h, M, r, false, d.on(), pair);
  float* T = T_save ? T_save : w.T;
  float* small_acc = nullptr;
  ZeroList zl;
  if (M <= kSmallMMax) {
    small_acc = y_dtype == QLORA_DTYPE_F32 ? static_cast<float*>(Y) : w.Yacc;
    zl.ptr[0] = small_acc;
    zl.len[0] = M * o;
  }
  if (M <= kDecodeMMax) {
    // Decode path, two launches: the split-K rank-r kernel zeroes the fp32
    // accumulator and writes the per-CTA partials of T = X L1; the decode
    // kernel streams the weight, sums the partials and adds the LoRA term.
    const int rows = rank_r_rows(r);
    const int64_t n_part = (h + rows - 1) / rows;
    {
      LaunchScope ls(QLORA_KERNEL_TGEMM, st);
      rank_r_small_kernel<<<static_cast<unsigned>(n_part), 256, 0, st>>>(
          static_cast<const uint16_t*>(X), static_cast<int>(M), h, static_cast<const uint16_t*>(L1), r, nullptr,
          w.P, small_acc, M * o, d.thr, d.seed, d.scale);
    }
    if (launch_status() != QLORA_OK) return QLORA_ERR_CUDA;
    CUtensorMap mc, mx;
    // codes as bytes [o][h/2]: one unit = 128 rows x 128 bytes, 128-byte swizzle
    if (!map_u8(&mc, Wq->codes, h / 2, o, h / 2, SD_UNIT_K / 2, SK_BN, CU_TENSOR_MAP_SWIZZLE_128B))
      return QLORA_ERR_CUDA;
    // tokens as [M][h/64][64]: one unit's slice = box {64, 4, M}, 128-byte swizzle
    if (!map_bf16_3d(&mx, X, 64, h / 64, M, 128, h * 2, 64, SD_UNIT_BLOCKS, static_cast<uint32_t>(M)))
      return QLORA_ERR_CUDA;
    DecodeParams dp{};
    dp.M = static_cast<int>(M);
    dp.N = static_cast<int>(o);
    dp.k_units = static_cast<int>((h + SD_UNIT_K - 1) / SD_UNIT_K);
    dp.blocks_per_row = static_cast<int>(h / 64);
    dp.r = r;
    dp.s = s;
    dp.units = ((o + SK_BN - 1) / SK_BN) * dp.k_units;
    dp.slot_bytes = static_cast<int>(((SD_CODE_BYTES + M * SD_UNIT_BLOCKS * SD_X_ROW_BYTES) + 1023) / 1024 * 1024);
    dp.low_bytes = static_cast<int>(((SD_BAR_BYTES + M * r * 4) + 1023) / 1024 * 1024);
    dp.P = w.P;
    dp.n_part = static_cast<int>(n_part);
    dp.T_out = T_save;
    dp.L2 = static_cast<const uint16_t*>(L2);
    dp.absmax_fp8 = Wq->absmax_fp8;
    dp.dq_scale = Wq->dq_scale;
    dp.dq_mean = Wq->dq_mean;
    dp.absmax32 = Wq->absmax;
    dp.out = small_acc;
    std::memcpy(dp.codebook, Wq->codebook, sizeof(dp.codebook));
    const int64_t grid = dp.units < sm_count() ? dp.units : sm_count();
    auto launch = [&](auto kernel) {
      if (set_smem(kernel, SD_SMEM_BYTES) != QLORA_OK) return QLORA_ERR_CUDA;
      LaunchScope ls(QLORA_KERNEL_SMALL_M, st);
      // programmatic dependent launch: the kernel's prologue overlaps the
      // rank-r kernel, whose results it waits for with griddepcontrol.wait
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(static_cast<unsigned>(grid));
      cfg.blockDim = dim3(SD_THREADS);
      cfg.dynamicSmemBytes = SD_SMEM_BYTES;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, kernel, mc, mx, dp) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
    };
    rc = M <= 8 ? launch(small_m_mma_kernel<1>) : launch(small_m_mma_kernel<2>);
    if (rc != QLORA_OK) return rc;
    if (y_dtype == QLORA_DTYPE_BF16) {
      LaunchScope ls(QLORA_KERNEL_AUX, st);
      f32_to_bf16_kernel<<<grid_for(M * o, 256, sm_count() * 4), 256, 0, st>>>(small_acc, M * o,
                                                                               static_cast<uint16_t*>(Y));
    }
    return launch_status();
  }
  rc = lora_prep(Wq, X, M, L1, L2, r, w, T, true, zl, st, M <= kSmallMMax, d);
  if (rc != QLORA_OK) return rc;
  rc = lora_split(T, w.TT, nullptr, nullptr, M, r, s, st);
  if (rc != QLORA_OK) return rc;

  const int rp = ((r + 63) / 64) * 64;
  const int KL = 2 * rp;
  if (M <= kSmallMMax) {
    // Small-M (decode) path: weights as the 128-row MMA operand, tokens as N.
    const int nmma = static_cast<int>(((M + 15) / 16) * 16);
    float* acc = small_acc;
    CUtensorMap mx, mc, ml2, mtt;
    if (!map_bf16(&mx, X, h, M, h * 2, 64, nmma)) return QLORA_ERR_CUDA;
    // codes as bytes [o][h/2]: one unit = 128 rows x 32 bytes, 32-byte swizzle (conflict-free row reads)
    if (!map_u8(&mc, Wq->codes, h / 2, o, h / 2, 32, SK_BN, CU_TENSOR_MAP_SWIZZLE_32B)) return QLORA_ERR_CUDA;
    if (!map_bf16(&ml2, w.L2x, KL, o, static_cast<uint64_t>(KL) * 2, 64, SK_BN)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mtt, w.TT, KL, M, static_cast<uint64_t>(KL) * 2, 64, nmma)) return QLORA_ERR_CUDA;
    SmallMParams sp{};
    sp.M = static_cast<int>(M);
    sp.N = static_cast<int>(o);
    sp.nmma = nmma;
    sp.k_units = static_cast<int>(h / SK_BK);
    sp.ext_units = KL / SK_BK;
    sp.blocks_per_row = static_cast<int>(h / 64);
    const int64_t tiles = (o + SK_BN - 1) / SK_BN;
    sp.units = tiles * (sp.k_units + sp.ext_units);
    sp.absmax_fp8 = Wq->absmax_fp8;
    sp.dq_scale = Wq->dq_scale;
    sp.dq_mean = Wq->dq_mean;
    sp.absmax32 = Wq->absmax;
    sp.out = acc;
    std::memcpy(sp.codebook, Wq->codebook, sizeof(sp.codebook));
    const int64_t grid = sp.units < sm_count() ? sp.units : sm_count();
    if (set_smem(small_m_fwd_kernel, SK_SMEM_BYTES) != QLORA_OK) return QLORA_ERR_CUDA;
    {
      LaunchScope ls(QLORA_KERNEL_SMALL_M, st);
      small_m_fwd_kernel<<<static_cast<unsigned>(grid), SK_THREADS, SK_SMEM_BYTES, st>>>(mx, mc, ml2, mtt, sp);
    }
    if (y_dtype == QLORA_DTYPE_BF16) {
      LaunchScope ls(QLORA_KERNEL_AUX, st);
      f32_to_bf16_kernel<<<grid_for(M * o, 256, sm_count() * 4), 256, 0, st>>>(acc, M * o,
                                                                              static_cast<uint16_t*>(Y));
    }
    return launch_status();
  }
  if (pair) {
    // many tokens: W' once to bf16, then the pair-tile GEMM with the LoRA stages
    rc = dequant_into(Wq, w.Wd, QLORA_KERNEL_WPRIME, st);
    if (rc != QLORA_OK) return rc;
    return launch_pair_gemm<false>(X, M, h, w.Wd, o, h, w.TT, w.L2x, KL, Y, y_dtype == QLORA_DTYPE_BF16, w,
                                   QLORA_KERNEL_FUSED_FWD, st);
  }
  CUtensorMap ma, mae, mbe, mc;
  if (!map_bf16(&ma, X, h, M, h * 2, 64, 256)) return QLORA_ERR_CUDA;
  if (!map_bf16(&mae, w.TT, KL, M, static_cast<uint64_t>(KL) * 2, 64, 256)) return QLORA_ERR_CUDA;
  if (!map_bf16(&mbe, w.L2x, KL, o, static_cast<uint64_t>(KL) * 2, 64, 256)) return QLORA_ERR_CUDA;
  // codes as bytes [o][h/2]: one stage = 256 rows x 32 bytes (one 64-block per row)
  if (!map_u8(&mc, Wq->codes, h / 2, o, h / 2, 32, 256)) return QLORA_ERR_CUDA;
  QGemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(o);
  p.k_main_stages = static_cast<int>(h / 64);
  p.k_ext_stages = KL / 64;
  p.blocks_per_row = static_cast<int>(h / 64);
  p.absmax_fp8 = Wq->absmax_fp8;
  p.dq_scale = Wq->dq_scale;
  p.dq_mean = Wq->dq_mean;
  p.absmax32 = Wq->absmax;
  p.out = Y;
  p.out_bf16 = y_dtype == QLORA_DTYPE_BF16;
  p.ld_out = o;
  std::memcpy(p.codebook, Wq->codebook, sizeof(p.codebook));
  if (set_smem(qgemm_nf4_kernel<false>, QG_SMEM_BYTES) != QLORA_OK) return QLORA_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((o + QG_BN - 1) / QG_BN), static_cast<unsigned>((M + QG_BM - 1) / QG_BM));
  {
    LaunchScope ls(QLORA_KERNEL_FUSED_FWD, st);
    qgemm_nf4_kernel<false><<<grid, QG_THREADS, QG_SMEM_BYTES, st>>>(ma, mae, mbe, mc, p);
  }
  return launch_status();
}

}  // namespace

namespace {

int linear_bwd_impl(const qlora_nf4_t* Wq, const void* X, const void* dY, int64_t M, const void* L1, const void* L2,
                    int r, float s, const DropoutCfg& d, const float* T_saved, void* dX, int dx_dtype, float* dL1,
                    float* dL2, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_linear_args(Wq, M, r, dx_dtype);
  if (rc != QLORA_OK) return rc;
  if (!X || !dY || !L1 || !L2 || !dX || !dL1 || !dL2) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(L1) || !aligned16(L2) || !aligned16(dX) || !aligned16(dL1) ||
      !aligned16(dL2) || (T_saved && !aligned16(T_saved)) || (ws && !aligned16(ws)))
    return QLORA_ERR_ALIGN;
  const int64_t o = Wq->o, h = Wq->h;
  if (!ws || ws_bytes < lora_ws_layout(nullptr, o, h, M, r, true, d.on()).bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pair = M >= kPairMMin && ws_bytes >= lora_ws_layout(nullptr, o, h, M, r, true, d.on(), true).bytes;
  const LoraWs w = lora_ws_layout(ws, o, h, M, r, true, d.on(), pair);
  const int rp = ((r + 63) / 64) * 64;
  const int KL = 2 * rp;

  // L1x, L2x, zeroed accumulators (U, dL1, dL2, and T when it is recomputed).
  float* T = T_saved ? const_cast<float*>(T_saved) : w.T;
  ZeroList zl;
  zl.ptr[0] = w.U;
  zl.len[0] = M * r;
  zl.ptr[1] = dL1;
  zl.len[1] = h * r;
  zl.ptr[2] = dL2;
  zl.len[2] = static_cast<int64_t>(r) * o;
  rc = lora_prep(Wq, X, M, L1, L2, r, w, T, T_saved == nullptr, zl, st, false, d);
  if (rc != QLORA_OK) return rc;
  if (d.on() && T_saved) {
    // the masked adapter input for dL1 (lora_prep builds it only to recompute T)
    LaunchScope ls(QLORA_KERNEL_AUX, st);
    const int64_t nvec = M * h / 8;
    dropout_mask_kernel<<<static_cast<unsigned>(grid_for(nvec, 256, sm_count() * 8)), 256, 0, st>>>(
        static_cast<const uint4*>(X), nvec, reinterpret_cast<uint4*>(w.Xm), d.thr, d.seed);
  }

  // U = dY L2^T: A = dY K-major [M][o]; B(n=j, k=i) = L2x[i][j], MN-major.
  {
    CUtensorMap ma, mb;
    if (!map_bf16(&ma, dY, o, M, o * 2, 64, 128)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb, w.L2x, rp, o, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    rc = launch_tgemm<false, true>(ma, mb, mb, static_cast<int>(M), r, static_cast<int>(o), false, w.U, r, false, st);
    if (rc != QLORA_OK) return rc;
    // s U -> UU and s T -> TT in one launch
    rc = lora_split(w.U, w.UU, T, w.TT, M, r, s, st);
    if (rc != QLORA_OK) return rc;
  }

  // dX = dY W'^T + [sU_hi | sU_lo] [L1 | L1]^T
  {
    // With dropout the LoRA term is masked per element of dX, so it cannot share
    // the accumulator: the GEMM computes dY W'^T alone (in fp32) and the masked
    // term is added below.
    float* dx32 = d.on() ? (dx_dtype == QLORA_DTYPE_F32 ? static_cast<float*>(dX) : w.dXf) : nullptr;
    void* gemm_out = d.on() ? static_cast<void*>(dx32) : dX;
    const int gemm_bf16 = !d.on() && dx_dtype == QLORA_DTYPE_BF16;
    if (pair) {
      // many tokens: W' once to bf16, then the pair-tile GEMM (W'^T as the MN-major operand)
      if (dequant_into(Wq, w.Wd, QLORA_KERNEL_WPRIME, st) != QLORA_OK) return QLORA_ERR_CUDA;
      if (launch_pair_gemm<true>(dY, M, o, w.Wd, o, h, w.UU, w.L1x, d.on() ? 0 : KL, gemm_out, gemm_bf16, w,
                                 QLORA_KERNEL_FUSED_BWD, st) != QLORA_OK)
        return QLORA_ERR_CUDA;
    } else {
      CUtensorMap ma, mae, mbe, mc;
      if (!map_bf16(&ma, dY, o, M, o * 2, 64, 256)) return QLORA_ERR_CUDA;
      if (!map_bf16(&mae, w.UU, KL, M, static_cast<uint64_t>(KL) * 2, 64, 256)) return QLORA_ERR_CUDA;
      if (!map_bf16(&mbe, w.L1x, KL, h, static_cast<uint64_t>(KL) * 2, 64, 256)) return QLORA_ERR_CUDA;
      // codes as bytes [o][h/2]: one stage = 64 rows (K) x 128 bytes (256 outputs along h)
      if (!map_u8(&mc, Wq->codes, h / 2, o, h / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
      QGemmParams p{};
      p.M = static_cast<int>(M);
      p.N = static_cast<int>(h);
      p.k_main_stages = static_cast<int>(o / 64);
      p.k_ext_stages = d.on() ? 0 : KL / 64;
      p.blocks_per_row = static_cast<int>(h / 64);
      p.absmax_fp8 = Wq->absmax_fp8;
      p.dq_scale = Wq->dq_scale;
      p.dq_mean = Wq->dq_mean;
      p.absmax32 = Wq->absmax;
      p.out = gemm_out;
      p.out_bf16 = gemm_bf16;
      p.ld_out = h;
      std::memcpy(p.codebook, Wq->codebook, sizeof(p.codebook));
      if (set_smem(qgemm_nf4_kernel<true>, QG_SMEM_BYTES) != QLORA_OK) return QLORA_ERR_CUDA;
      dim3 grid(static_cast<unsigned>((h + QG_BN - 1) / QG_BN), static_cast<unsigned>((M + QG_BM - 1) / QG_BM));
      {
        LaunchScope ls(QLORA_KERNEL_FUSED_BWD, st);
        qgemm_nf4_kernel<true><<<grid, QG_THREADS, QG_SMEM_BYTES, st>>>(ma, mae, mbe, mc, p);
      }
      if (launch_status() != QLORA_OK) return QLORA_ERR_CUDA;
    }
    if (d.on()) {
      // dX += scale * keep * ([sU_hi | sU_lo] [L1 | L1]^T): rows = tokens, cols = h, K = the packed rank
      CUtensorMap mu, ml;
      if (!map_bf16(&mu, w.UU, KL, M, static_cast<uint64_t>(KL) * 2, 64, TG_BM)) return QLORA_ERR_CUDA;
      if (!map_bf16(&ml, w.L1x, KL, h, static_cast<uint64_t>(KL) * 2, 64, 256)) return QLORA_ERR_CUDA;
      rc = launch_tgemm<false, false>(mu, ml, ml, static_cast<int>(M), static_cast<int>(h), KL, false, dx32, h,
                                      false, st, d.scale, &d, h);
      if (rc != QLORA_OK) return rc;
      if (dx_dtype == QLORA_DTYPE_BF16) {
        LaunchScope ls(QLORA_KERNEL_AUX, st);
        f32_to_bf16_kernel<<<grid_for(M * h, 256, sm_count() * 4), 256, 0, st>>>(dx32, M * h,
                                                                                 static_cast<uint16_t*>(dX));
        if (launch_status() != QLORA_OK) return QLORA_ERR_CUDA;
      }
    }
  }

  // dL1 = X^T (sU) with sU = hi + lo:  rows i of h, cols j of r, K = tokens
  // (with dropout: scale (X * keep)^T (sU)).
  {
    CUtensorMap ma, mb, mb2;
    if (!map_bf16(&ma, d.on() ? static_cast<const void*>(w.Xm) : X, h, M, h * 2, 64, 64)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb, w.UU, rp, M, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb2, w.UU + rp, rp, M, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    rc = launch_tgemm<true, true>(ma, mb, mb2, static_cast<int>(h), r, static_cast<int>(M), true, dL1, r, false, st,
                                  d.scale);
    if (rc != QLORA_OK) return rc;
  }

  // dL2 = (sT)^T dY, computed as dL2^T = dY^T (sT): rows = o, cols = r, stored transposed.
  {
    CUtensorMap ma, mb, mb2;
    if (!map_bf16(&ma, dY, o, M, o * 2, 64, 64)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb, w.TT, rp, M, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    if (!map_bf16(&mb2, w.TT + rp, rp, M, static_cast<uint64_t>(KL) * 2, 64, 64)) return QLORA_ERR_CUDA;
    rc = launch_tgemm<true, true>(ma, mb, mb2, static_cast<int>(o), r, static_cast<int>(M), true, dL2, o, true, st);
    if (rc != QLORA_OK) return rc;
  }
  return QLORA_OK;
}

// p in [0, 1) -> the keep threshold floor(p 2^32) and the fp32 scale 1 / (1 - p).
bool make_dropout(float p, uint64_t seed, DropoutCfg* d) {
  if (!(p >= 0.0f && p < 1.0f)) return false;
  const double t = std::floor(static_cast<double>(p) * 4294967296.0);
  d->thr = t >= 4294967295.0 ? 0xFFFFFFFFu : static_cast<uint32_t>(t);
  d->seed = seed;
  volatile float one_minus = 1.0f - p;  // fp32 operations, no contraction
  d->scale = 1.0f / one_minus;
  if (d->thr == 0) d->scale = 1.0f;   // p < 2^-32: nothing can be dropped
  return true;
}

}  // namespace

extern "C" {

int qlora_linear_fwd(const qlora_nf4_t* Wq, const void* X, int64_t M, const void* L1, const void* L2, int r, float s,
                     void* Y, int y_dtype, float* T_save, void* ws, size_t ws_bytes, void* stream) {
  return linear_fwd_impl(Wq, X, M, L1, L2, r, s, DropoutCfg(), Y, y_dtype, T_save, ws, ws_bytes, stream);
}

int qlora_linear_bwd(const qlora_nf4_t* Wq, const void* X, const void* dY, int64_t M, const void* L1, const void* L2,
                     int r, float s, const float* T_saved, void* dX, int dx_dtype, float* dL1, float* dL2, void* ws,
                     size_t ws_bytes, void* stream) {
  return linear_bwd_impl(Wq, X, dY, M, L1, L2, r, s, DropoutCfg(), T_saved, dX, dx_dtype, dL1, dL2, ws, ws_bytes,
                         stream);
}

size_t qlora_linear_fwd_dropout_workspace_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, false, true, true).bytes;
}

size_t qlora_linear_bwd_dropout_workspace_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, true, true, true).bytes;
}

size_t qlora_linear_fwd_dropout_workspace_min_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, false, true).bytes;
}

size_t qlora_linear_bwd_dropout_workspace_min_size(int64_t o, int64_t h, int64_t M, int r) {
  return lora_ws_layout(nullptr, o, h, M, r, true, true).bytes;
}

int qlora_linear_fwd_dropout(const qlora_nf4_t* Wq, const void* X, int64_t M, const void* L1, const void* L2, int r,
                             float s, float p, uint64_t seed, void* Y, int y_dtype, float* T_save, void* ws,
                             size_t ws_bytes, void* stream) {
  DropoutCfg d;
  if (!make_dropout(p, seed, &d)) return QLORA_ERR_UNSUPPORTED;
  return linear_fwd_impl(Wq, X, M, L1, L2, r, s, d, Y, y_dtype, T_save, ws, ws_bytes, stream);
}

int qlora_linear_bwd_dropout(const qlora_nf4_t* Wq, const void* X, const void* dY, int64_t M, const void* L1,
                             const void* L2, int r, float s, float p, uint64_t seed, const float* T_saved, void* dX,
                             int dx_dtype, float* dL1, float* dL2, void* ws, size_t ws_bytes, void* stream) {
  DropoutCfg d;
  if (!make_dropout(p, seed, &d)) return QLORA_ERR_UNSUPPORTED;
  return linear_bwd_impl(Wq, X, dY, M, L1, L2, r, s, d, T_saved, dX, dx_dtype, dL1, dL2, ws, ws_bytes, stream);
}

int qlora_paged_alloc(size_t bytes, void** ptr) {
  if (!ptr) return QLORA_ERR_NULL;
  *ptr = nullptr;
  if (bytes == 0) return QLORA_ERR_SHAPE;
  void* q = nullptr;
  if (cudaMallocManaged(&q, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  *ptr = q;
  return QLORA_OK;
}

int qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int qlora_paged_advise(void* ptr, size_t bytes, int prefer_host) {
  if (!ptr) return QLORA_ERR_NULL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  const int where = prefer_host ? cudaCpuDeviceId : dev;
  if (cudaMemAdvise(ptr, bytes, cudaMemAdviseSetPreferredLocation, where) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemAdvise(ptr, bytes, cudaMemAdviseSetAccessedBy, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

int qlora_paged_prefetch(void* ptr, size_t bytes, int to_host, void* stream) {
  if (!ptr) return QLORA_ERR_NULL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  return cudaMemPrefetchAsync(ptr, bytes, to_host ? cudaCpuDeviceId : dev, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

int qlora_grad_sqnorm(const float* g, int64_t n, double* acc, void* stream) {
  if (!g || !acc) return QLORA_ERR_NULL;
  if (n <= 0) return QLORA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(acc) & 7u) != 0) return QLORA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    LaunchScope ls(QLORA_KERNEL_OPTIM, st);
    grad_sqnorm_kernel<<<static_cast<unsigned>(grid_for(n / 4 + 1, 256 * 4, sm_count() * 4)), 256, 0, st>>>(g, n,
                                                                                                          acc);
  }
  return launch_status();
}

int qlora_adamw_step(float* param, const float* grad, float* m, float* v, uint16_t* param_bf16, int64_t n,
                     const qlora_adamw_t* hp, const double* sqnorm, void* stream) {
  if (!param || !grad || !m || !v || !hp) return QLORA_ERR_NULL;
  if (n <= 0 || hp->step < 1) return QLORA_ERR_SHAPE;
  if (!(hp->beta1 >= 0.0f && hp->beta1 < 1.0f && hp->beta2 >= 0.0f && hp->beta2 < 1.0f && hp->eps > 0.0f &&
        hp->lr >= 0.0f && hp->weight_decay >= 0.0f && (!sqnorm || hp->max_grad_norm > 0.0f)))
    return QLORA_ERR_UNSUPPORTED;
  AdamWParams a{};
  a.lr = hp->lr;
  a.beta1 = hp->beta1;
  a.beta2 = hp->beta2;
  a.eps = hp->eps;
  a.weight_decay = hp->weight_decay;
  // bias corrections in double, rounded once to fp32
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  a.step_size = static_cast<float>(static_cast<double>(hp->lr) / bc1);
  a.bc2_sqrt = static_cast<float>(std::sqrt(bc2));
  a.max_grad_norm = hp->max_grad_norm;
  a.sqnorm = sqnorm;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    LaunchScope ls(QLORA_KERNEL_OPTIM, st);
    adamw_kernel<<<static_cast<unsigned>(grid_for(n, 256 * 4, sm_count() * 8)), 256, 0, st>>>(param, grad, m, v,
                                                                                             param_bf16, n, a);
  }
  return launch_status();
}

int qlora_merge_bf16(const qlora_nf4_t* Wq, const void* L1, const void* L2, int r, float s, void* out,
                     void* stream) {
  const int rc = check_wq(Wq);
  if (rc != QLORA_OK) return rc;
  if (!L1 || !L2 || !out) return QLORA_ERR_NULL;
  if (r < 8 || r > QLORA_MAX_RANK || r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (Wq->o % 64 != 0 || Wq->o > (int64_t(1) << 30) || Wq->h > (int64_t(1) << 30)) return QLORA_ERR_SHAPE;
  if (!aligned16(L1) || !aligned16(L2) || !aligned16(out)) return QLORA_ERR_ALIGN;
  const int64_t o = Wq->o, h = Wq->h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap ml2, ml1;
  // A = L2^T: L2 [r][o] read as MN-major tiles {64 n, 64 ranks}; B = L1 [h][r], K-major {64 ranks, 256 k}
  if (!map_bf16(&ml2, L2, o, r, o * 2, 64, 64)) return QLORA_ERR_CUDA;
  if (!map_bf16(&ml1, L1, r, h, static_cast<uint64_t>(r) * 2, 64, MG_BN)) return QLORA_ERR_CUDA;
  MergeParams p{};
  p.o = static_cast<int>(o);
  p.h = static_cast<int>(h);
  p.k_stages = (r + 63) / 64;
  p.s = s;
  p.codes = Wq->codes;
  p.absmax_fp8 = Wq->absmax_fp8;
  p.dq_scale = Wq->dq_scale;
  p.dq_mean = Wq->dq_mean;
  p.absmax32 = Wq->absmax;
  p.out = static_cast<uint16_t*>(out);
  std::memcpy(p.codebook, Wq->codebook, sizeof(p.codebook));
  int smem = p.k_stages * (MG_A_STAGE + MG_B_STAGE) + 1024 + 64;
  if (smem < MG_MIN_SMEM) smem = MG_MIN_SMEM;
  if (set_smem(merge_kernel, smem) != QLORA_OK) return QLORA_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((o + MG_BM - 1) / MG_BM), static_cast<unsigned>((h + MG_BN - 1) / MG_BN));
  {
    LaunchScope ls(QLORA_KERNEL_MERGE, st);
    merge_kernel<<<grid, MG_THREADS, smem, st>>>(ml2, ml1, p);
  }
  return launch_status();
}

void qlora_trace_enable(int on) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  t.on = on != 0;
  for (const TraceRec& r : t.recs) {
    t.pool.push_back(r.start);
    t.pool.push_back(r.stop);
  }
  t.recs.clear();
}

int qlora_trace_read(int family, double* total_ms, int64_t* launches) {
  if (!total_ms || !launches) return QLORA_ERR_NULL;
  if (family < 0 || family >= QLORA_KERNEL_FAMILIES) return QLORA_ERR_UNSUPPORTED;
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  double ms = 0.0;
  int64_t n = 0;
  std::vector<TraceRec> keep;
  for (const TraceRec& r : t.recs) {
    if (r.family != family) {
      keep.push_back(r);
      continue;
    }
    float e = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&e, r.start, r.stop) != cudaSuccess)
      return QLORA_ERR_CUDA;
    ms += e;
    ++n;
    t.pool.push_back(r.start);
    t.pool.push_back(r.stop);
  }
  t.recs.swap(keep);
  *total_ms = ms;
  *launches = n;
  return QLORA_OK;
}

const char* qlora_kernel_family_name(int family) {
  switch (family) {
    case QLORA_KERNEL_QUANTIZE: return "nf4_quantize";
    case QLORA_KERNEL_DOUBLE_QUANT: return "double_quant";
    case QLORA_KERNEL_DEQUANT: return "nf4_dequant";
    case QLORA_KERNEL_FUSED_FWD: return "nf4_gemm_fwd";
    case QLORA_KERNEL_FUSED_BWD: return "nf4_gemm_bwd_dx";
    case QLORA_KERNEL_TGEMM: return "rank_r_gemm";
    case QLORA_KERNEL_AUX: return "lora_aux";
    case QLORA_KERNEL_SMALL_M: return "small_m_fwd";
    case QLORA_KERNEL_MERGE: return "adapter_merge";
    case QLORA_KERNEL_OPTIM: return "lora_optimizer";
    case QLORA_KERNEL_WPRIME: return "nf4_dequant_wprime";
    default: return "unknown";
  }
}

int64_t qlora_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ====================================================================== no-allocation forward

// Scratch of qlora_linear_fwd_noalloc.  Host code cannot use this name as a
// device address (on the host it is only a stand-in); the address is looked
// up per device with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" {

int qlora_linear_fwd_noalloc(const qlora_nf4_t* Wq, const void* X, int64_t M, const void* L1, const void* L2, int r,
                             float s, void* Y, int y_dtype, float* T_save, void* stream) {
  const int rc = check_linear_args(Wq, M, r, y_dtype);
  if (rc != QLORA_OK) return rc;
  if (qlora_linear_fwd_workspace_min_size(Wq->o, Wq->h, M, r) > QLORA_NOALLOC_SCRATCH_BYTES)
    return QLORA_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  const int sc = noalloc_scratch(&ws);
  if (sc != QLORA_OK) return sc;
  return qlora_linear_fwd(Wq, X, M, L1, L2, r, s, Y, y_dtype, T_save, ws, QLORA_NOALLOC_SCRATCH_BYTES, stream);
}

unsigned int qlora_debug_wait_tags(void) {
  unsigned int tags = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return 0xFFFFFFFFu;
  if (cudaMemcpyFromSymbol(&tags, g_wait_tags, sizeof(tags)) != cudaSuccess) return 0xFFFFFFFFu;
  const unsigned int zero = 0;
  cudaMemcpyToSymbol(g_wait_tags, &zero, sizeof(zero));
  return tags;
}

int qlora_debug_wait_probe(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return QLORA_ERR_UNSUPPORTED;
  {
    LaunchScope ls(QLORA_KERNEL_AUX, static_cast<cudaStream_t>(stream));
    wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns));
  }
  return launch_status();
}

int qlora_check_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_status, sizeof(h)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (h != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
    return (h & kStatusTimeout) ? QLORA_ERR_TIMEOUT : QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

}  // extern "C"
