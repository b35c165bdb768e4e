// C ABI of libqlora: argument validation, TMA tensor maps, workspace layout,
// split planning and the launch sequence of every entry point in qlora.h.
// All device work is enqueued on the caller's stream; nothing here allocates
// device memory or synchronises (except qlora_last_device_status and
// qlora_trace_end, which say so).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <vector>

#include "../../include/qlora.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace ql {
// kernels implemented in the other translation units
cudaError_t launch_nf4_quantize(const bf16* w, int64_t numel, uint8_t* codes, float* absmax, cudaStream_t st);
cudaError_t launch_nf4_dequantize(const uint8_t* const* codes, const float* const* absmax, const int64_t* numel,
                                  bf16* const* out, int n, cudaStream_t st, int num_sms);
cudaError_t launch_gemm_nf4(int mode, int epi, int tiles, const GemmMaps& maps, const GemmArgs& args,
                            cudaStream_t stream);
int gemm_nf4_b_cols_per_cta(int tiles);
cudaError_t launch_rowproj(int rw, int nf, bool bt, const CUtensorMap& t, const CUtensorMap& v0,
                           const CUtensorMap& v1, const CUtensorMap& v2, const ReduceJob& job, int nkc, int* status,
                           cudaStream_t st);
cudaError_t launch_colproj(int R, int cc, const CUtensorMap& t, const CUtensorMap& u, const ReduceJob& job, int nmc,
                           int nch, int* status, cudaStream_t st);
int colproj_chunks(int R);  // the widest colproj unit (column chunks of 64) for a tile width R
cudaError_t launch_dypass(const CUtensorMap& t, const CUtensorMap& u, const CUtensorMap& b, const ReduceJob& gjob,
                          const ReduceJob& qjob, int nch, int* status, cudaStream_t st);
cudaError_t arm_inject_timeout();
cudaError_t launch_reduce(const ReduceJob* jobs, int n, cudaStream_t st);
cudaError_t launch_rmsnorm_fwd(const bf16* X, const bf16* w, int M, int d, float eps, int plus_one, bf16* Y,
                               float* rstd, cudaStream_t st);
cudaError_t launch_rmsnorm_bwd(const bf16* X, const bf16* w, const float* rstd, const bf16* dY, int M, int d,
                               int plus_one, bf16* dX, cudaStream_t st);
extern const uint32_t h_nf4_bits[16];
int g_grid_cap = 0;
}  // namespace ql

using namespace ql;

namespace {

// ------------------------------------------------------------- tracing ---
enum KernelId : int {
  K_QUANT = 0, K_DEQUANT, K_GEMM_FWD, K_GEMM_GLU_FWD, K_GEMM_BWD, K_GEMM_GLU_BWD, K_ROWPROJ, K_COLPROJ, K_DYPASS,
  K_REDUCE, K_NORM_FWD, K_NORM_BWD, K_COUNT
};
const char* const kKernelNames[K_COUNT] = {
    "nf4_quantize", "nf4_dequantize", "gemm_nf4_fwd", "gemm_nf4_gateup_glu_fwd", "gemm_nf4_bwd_dx",
    "gemm_nf4_down_bwd_glu", "skinny_rowproj", "skinny_colproj", "skinny_dypass", "skinny_reduce", "rmsnorm_fwd", "rmsnorm_bwd"};

std::atomic<uint64_t> g_launches{0};
bool g_trace = false;
int g_trace_only = -1;  // kernel id traced alone (qlora_trace_begin_only), -1 = every kernel
struct TraceRec {
  int id;
  cudaEvent_t a, b;
};
std::vector<TraceRec> g_recs;
std::vector<cudaEvent_t> g_pool;
size_t g_pool_used = 0;
int32_t g_tiles = 0;  // GEMM tile configuration (see qlora_set_tile_config); 0 = automatic
// Automatic choice: the gated-MLP calls with at most this many tokens dequantise in the
// GEMM mainloop (configuration 2), where that beats decoding the three weights once into
// staging buffers (configuration 4); measured on the Llama-7B MLP: 0.441 vs 0.495 ms per
// fwd+bwd at 256 tokens, 0.531 vs 0.547 at 512, 0.668 vs 0.641 at 1024.
constexpr int64_t kAutoMainloopMaxM = 512;
#ifndef QL_GROUP_M
#define QL_GROUP_M 8
#endif
constexpr int kGroupM = QL_GROUP_M;  // output-row tiles per group of the GEMM tile order
// Largest M, k_in, n_out (and nq + nk + nv) a call accepts.  The skinny
// reductions index rows x factor columns (up to 192) and the GEMMs count
// output tiles in 32-bit integers; at 2^23 both stay below 2^31.
constexpr int64_t kMaxDim = int64_t(1) << 23;

// Internal view of one projection: a frozen NF4 base (codes + absmax) or a
// frozen bf16 base (w16), plus its LoRA factors.
struct Wt {
  const uint8_t* codes;
  const float* absmax;
  const qlora_bf16* w16;
  int64_t n_out, k_in;
};
struct Lin {
  Wt w;
  const qlora_bf16* A;
  const qlora_bf16* B;
  int32_t r;
  float scale;
};
Lin lin_of(const qlora_lora_linear& l) { return {{l.w.codes, l.w.absmax, nullptr, l.w.n_out, l.w.k_in}, l.A, l.B, l.r, l.scale}; }
Lin lin_of(const qlora_lora_linear16& l) { return {{nullptr, nullptr, l.w, l.n_out, l.k_in}, l.A, l.B, l.r, l.scale}; }

cudaEvent_t pool_event() {
  if (g_pool_used == g_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_pool.push_back(e);
  }
  return g_pool[g_pool_used++];
}

struct KScope {
  int id;
  cudaStream_t st;
  cudaEvent_t b = nullptr;
  KScope(int id_, cudaStream_t st_) : id(id_), st(st_) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_trace && (g_trace_only < 0 || g_trace_only == id)) {
      cudaEvent_t a = pool_event();
      b = pool_event();
      if (a && b) {
        cudaEventRecord(a, st);
        g_recs.push_back({id, a, b});
      } else {
        b = nullptr;
      }
    }
  }
  ~KScope() {
    if (b) cudaEventRecord(b, st);
  }
};

// ------------------------------------------------------------ helpers ---
int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Backward of an empty batch (M = 0): every adapter gradient is a sum over no
// tokens, so it is zero.  The gradients are cleared on the stream (a data-
// parallel all-reduce then sums correct values from a rank whose shard is
// empty); nothing else is read or written.
qlora_status zero_adapter_grads(qlora_bf16* const* g, const int64_t* elems, int n, cudaStream_t st) {
  for (int i = 0; i < n; ++i) {
    if (!g[i]) return QLORA_ERR_INVALID_ARG;
    if (misaligned(g[i])) return QLORA_ERR_MISALIGNED;
  }
  for (int i = 0; i < n; ++i)
    if (cudaMemsetAsync(g[i], 0, static_cast<size_t>(elems[i]) * sizeof(qlora_bf16), st) != cudaSuccess)
      return QLORA_ERR_CUDA;
  return QLORA_OK;
}
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] matrix with `ld` elements per row.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, int64_t cols, int64_t rows,
              int64_t ld, int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool map_bf16(CUtensorMap* m, const void* p, int64_t cols, int64_t rows, int64_t ld, int bc, int br,
              CUtensorMapSwizzle s) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, cols, rows, ld, bc, br, s);
}

// ---------------------------------------------------------- planning ----
// Skinny passes run up to four persistent CTAs per SM; a CTA's ring holds four
// stages of one 64x64 tile of T plus 128 bytes per factor column (the grid
// shrinks when wide factor tiles limit residency).
int skinny_target_ctas(int factor_cols) {
  const int smem = 4 * (8192 + 128 * factor_cols) + 64 + 1024;
  // the device's SMs (148 when none is present)
  return apply_grid_cap(num_sms() * std::max(1, std::min(4, 232448 / smem)), 1);
}

// Partition of `groups` output groups of `upg` units each over the CTAs:
// unit granularity while there are fewer groups than CTAs (every CTA streams
// the same number of tiles), whole groups otherwise (one partial per group).
struct SkPlan {
  SkPart sp;
  int slot_cap;
};
SkPlan plan_skinny(int64_t groups, int64_t upg, int target) {
  SkPlan p;
  const int64_t units = groups * upg;
  int64_t align = groups >= target ? upg : 1;
  while (cdiv(units, align) > (int64_t(1) << 30)) align *= 2;  // keep the unit count in int range
  const int64_t U = cdiv(units, align);
  p.sp.U = static_cast<int>(U);
  p.sp.P = static_cast<int>(std::min<int64_t>(target, U));
  p.sp.align = static_cast<int>(align);
  p.sp.upg = static_cast<int>(upg);
  p.slot_cap = 1;
  for (int64_t g = 0; g < groups; ++g) p.slot_cap = std::max(p.slot_cap, sk_slots(p.sp, static_cast<int>(g)));
  return p;
}
constexpr int kDyCC = 4;  // column chunks of 64 per dypass unit (matches the kernel)
// rowproj: T [M, K] times factors of `fcols` columns in all; reduction over K (padded to 64)
// `target` > 0 overrides the CTA count (at most one CTA per 64-row group then
// gives every group a single partial slot).
SkPlan plan_rowproj(int64_t M, int64_t K, int fcols, int target = 0) {
  return plan_skinny(cdiv(M, 64), cdiv(K, 64), target > 0 ? target : skinny_target_ctas(fcols));
}
// colproj units of `cc` column chunks of 64 (R the factor-tile width).  Several chunks side by
// side read colproj_chunks(R) x 128 contiguous bytes of each row, which pays on wide operands, but
// every CTA then writes a partial that many times taller; one chunk is kept unless those partials
// stay within 1/16 of the bytes the pass streams.
int colproj_cc_for(int64_t M, int64_t ncols, int R) {
  const int cmax = colproj_chunks(R);
  const double partials = static_cast<double>(skinny_target_ctas(R)) * cmax * 64 * R * 4;
  return partials * 16 <= static_cast<double>(M) * ncols * 2 ? cmax : 1;
}
SkPlan plan_colproj(int64_t M, int64_t ncols, int R) {
  return plan_skinny(cdiv(cdiv(ncols, 64), colproj_cc_for(M, ncols, R)), cdiv(M, 64), skinny_target_ctas(R));
}
SkPlan plan_dypass(int64_t M, int64_t N) {
  return plan_skinny(cdiv(cdiv(N, 64), kDyCC), cdiv(M, 64), skinny_target_ctas(32));
}
size_t rowproj_part_bytes(int64_t M, int64_t K, int R, int target = 0) {
  return static_cast<size_t>(cdiv(M, 64)) * plan_rowproj(M, K, R, target).slot_cap * 64 * R * 4;
}
size_t colproj_part_bytes(int64_t M, int64_t ncols, int R) {
  R = R <= 16 ? 16 : (R <= 32 ? 32 : (R <= 64 ? 64 : 128));  // the kernel's tile width
  const int cc = colproj_cc_for(M, ncols, R);
  return static_cast<size_t>(cdiv(cdiv(ncols, 64), cc)) * plan_colproj(M, ncols, R).slot_cap * cc * 64 * R * 4;
}
size_t dypass_gpart_bytes(int64_t M, int64_t N) {
  return align256(static_cast<size_t>(cdiv(M, 64)) * cdiv(cdiv(N, 64), kDyCC) * 64 * 16 * 4);
}
// partials of the dY pass: fused for rank 16, a G pass then a dB pass for larger ranks
size_t dypass_part_bytes(int64_t M, int64_t N, int r) {
  if (r != 16) return std::max(rowproj_part_bytes(M, N, r), colproj_part_bytes(M, N, r));
  const int64_t ncb = cdiv(cdiv(N, 64), kDyCC);
  return dypass_gpart_bytes(M, N) + static_cast<size_t>(ncb) * plan_dypass(M, N).slot_cap * kDyCC * 64 * 16 * 4;
}
// Test hook (qlora_test_shrink_next_slot_cap): the next skinny pass whose plan
// gives some group more than one partial slot tells its kernels one slot fewer
// than the plan has (the partial buffer keeps the plan's size, so every access
// stays inside it).  The checked build's kernels then report QL_DEV_BAD_CONFIG.
int g_shrink_slot_cap = 0;
int planned_slot_cap(int cap) {
  if (g_shrink_slot_cap && cap > 1) {
    g_shrink_slot_cap = 0;
    return cap - 1;
  }
  return cap;
}

ReduceJob reduce_job(float* part, int64_t groups, int grows, int64_t rows, int R, int slot_cap, int nslots,
                     const SkPart& sp, const ReduceOuts& outs) {
  ReduceJob j;
  std::memset(&j, 0, sizeof(j));
  j.part = part;
  j.groups = static_cast<int>(groups);
  j.grows = grows;
  j.rows = static_cast<int>(rows);
  j.R = R;
  j.slot_cap = slot_cap;
  j.nslots = nslots;
  j.sp = sp;
  j.outs = outs;
  return j;
}

// ------------------------------------------------------------ passes ----
qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// A rank-side factor [rows, cols] (row stride ld) as the skinny kernels read it
// in tiles `tcols` wide (>= cols; the TMA zero-fills the difference): 64-row
// boxes of min(tcols, 64) columns in the swizzle of that row width.
bool map_factor(CUtensorMap* m, const void* p, int64_t rows, int cols, int64_t ld, int tcols = 0) {
  const int tc = tcols ? tcols : cols;
  const int subw = tc < 64 ? tc : 64;
  const CUtensorMapSwizzle swz = subw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                            : (subw == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  return map_bf16(m, p, cols, rows, ld, subw, 64, swz);
}

// Reductions collected for one launch: those of passes whose results nothing
// reads until later, each with its own partial region.
struct ReduceBatch {
  ReduceJob j[kMaxReduceJobs];
  int n = 0;
};
// Runs the reductions of a pass now, or appends them to `batch` (flush_reduce launches them).
qlora_status reduce_now_or_later(const ReduceJob* jobs, int n, ReduceBatch* batch, cudaStream_t st) {
  if (batch) {
    if (batch->n + n > kMaxReduceJobs) return QLORA_ERR_CUDA;  // planning error inside the library
    for (int i = 0; i < n; ++i) batch->j[batch->n++] = jobs[i];
    return QLORA_OK;
  }
  KScope k(K_REDUCE, st);
  return cuda_status(launch_reduce(jobs, n, st));
}
qlora_status flush_reduce(ReduceBatch& b, cudaStream_t st) {
  if (b.n == 0) return QLORA_OK;
  KScope k(K_REDUCE, st);
  const qlora_status s = cuda_status(launch_reduce(b.j, b.n, st));
  b.n = 0;
  return s;
}

// P = T V (V = up to three [K, r] LoRA A factors side by side) -> outs (bf16, optional scaled copies)
qlora_status pass_rowproj(const bf16* T, int64_t M, int64_t K, const bf16* V0, const bf16* V1, int r, float* part,
                          ReduceOuts outs, int* status, cudaStream_t st, const bf16* V2 = nullptr,
                          int target = 0) {
  CUtensorMap mt, mv0, mv1, mv2;
  const int nv = V2 ? 3 : (V1 ? 2 : 1);
  if (!map_bf16(&mt, T, K, M, K, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  if (!map_factor(&mv0, V0, K, r, r)) return QLORA_ERR_CUDA;
  if (!map_factor(&mv1, V1 ? V1 : V0, K, r, r)) return QLORA_ERR_CUDA;
  if (!map_factor(&mv2, V2 ? V2 : V0, K, r, r)) return QLORA_ERR_CUDA;
  const SkPlan p = plan_rowproj(M, K, nv * r, target);
  const int64_t nrc = cdiv(M, 64);
  ReduceJob j = reduce_job(part, nrc, 64, M, nv * r, planned_slot_cap(p.slot_cap), 0, p.sp, outs);
  j.status = status;
  {
    KScope k(K_ROWPROJ, st);
    const qlora_status s =
        cuda_status(launch_rowproj(r, nv, false, mt, mv0, mv1, mv2, j, (int)cdiv(K, 64), status, st));
    if (s != QLORA_OK) return s;
  }
  return reduce_now_or_later(&j, 1, nullptr, st);
}

// G = T B^T (B = LoRA right factor [r, N]) -> outs
qlora_status pass_rowproj_bt(const bf16* T, int64_t M, int64_t N, const bf16* B, int r, float* part,
                             ReduceOuts outs, int* status, cudaStream_t st, int64_t ldt = 0) {
  CUtensorMap mt, mb;
  if (!map_bf16(&mt, T, N, M, ldt ? ldt : N, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  if (!map_bf16(&mb, B, N, r, N, 64, r, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  const SkPlan p = plan_rowproj(M, N, r);
  const int64_t nrc = cdiv(M, 64);
  ReduceJob j = reduce_job(part, nrc, 64, M, r, planned_slot_cap(p.slot_cap), 0, p.sp, outs);
  j.status = status;
  {
    KScope k(K_ROWPROJ, st);
    const qlora_status s = cuda_status(launch_rowproj(r, 1, true, mt, mb, mb, mb, j, (int)cdiv(N, 64), status, st));
    if (s != QLORA_OK) return s;
  }
  return reduce_now_or_later(&j, 1, nullptr, st);
}

// Supported factor-tile widths of the colproj kernel: R rounded up to 16, 32, 64 or 128.
int colproj_width(int R) { return R <= 16 ? 16 : (R <= 32 ? 32 : (R <= 64 ? 64 : 128)); }

// Q = T^T U (U [M, R] with row stride ldu, R <= 128) -> outs
qlora_status pass_colproj(const bf16* T, int64_t M, int64_t ncols, const bf16* U, int R, float* part,
                          ReduceOuts outs, int* status, cudaStream_t st, int64_t ldt = 0, int64_t ldu = 0,
                          ReduceBatch* batch = nullptr) {
  CUtensorMap mt, mu;
  if (!map_bf16(&mt, T, ncols, M, ldt ? ldt : ncols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  if (!map_factor(&mu, U, M, R, ldu ? ldu : R, colproj_width(R))) return QLORA_ERR_CUDA;
  R = colproj_width(R);
  const SkPlan p = plan_colproj(M, ncols, R);
  const int cc = colproj_cc_for(M, ncols, R);
  const int64_t nch = cdiv(ncols, 64);
  ReduceJob j = reduce_job(part, cdiv(nch, cc), cc * 64, ncols, R, planned_slot_cap(p.slot_cap), 0, p.sp, outs);
  j.status = status;
  {
    KScope k(K_COLPROJ, st);
    const qlora_status s = cuda_status(launch_colproj(R, cc, mt, mu, j, (int)cdiv(M, 64), (int)nch, status, st));
    if (s != QLORA_OK) return s;
  }
  return reduce_now_or_later(&j, 1, batch, st);
}

// G = T Bl^T ([M, r]) and Q = T^T U ([N, r]) for T [M, N]: one fused read of T
// at rank 16 (its two reductions may go to `batch`), a G pass and a Q pass at
// larger ranks (which reuse `part`, so they are reduced at once).
qlora_status pass_dypass(const bf16* T, int64_t M, int64_t N, const bf16* U, const bf16* Bl, int r, float* part,
                         ReduceOuts gouts, ReduceOuts qouts, int* status, cudaStream_t st, int64_t ldt = 0,
                         int64_t ldu = 0, ReduceBatch* batch = nullptr) {
  if (r != 16) {
    const qlora_status s = pass_rowproj_bt(T, M, N, Bl, r, part, gouts, status, st, ldt);
    if (s != QLORA_OK) return s;
    return pass_colproj(T, M, N, U, r, part, qouts, status, st, ldt, ldu);
  }
  CUtensorMap mt, mu, mb;
  if (!map_bf16(&mt, T, N, M, ldt ? ldt : N, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  if (!map_factor(&mu, U, M, 16, ldu ? ldu : 16)) return QLORA_ERR_CUDA;
  if (!map_bf16(&mb, Bl, N, 16, N, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  const SkPlan p = plan_dypass(M, N);
  const int64_t nrc = cdiv(M, 64), nch = cdiv(N, 64), ncb = cdiv(nch, kDyCC);
  float* gpart = part;
  float* qpart = reinterpret_cast<float*>(reinterpret_cast<char*>(part) + dypass_gpart_bytes(M, N));
  ReduceJob jg = reduce_job(gpart, nrc, 64, M, 16, (int)ncb, (int)ncb, p.sp, gouts);
  ReduceJob jq = reduce_job(qpart, ncb, kDyCC * 64, N, 16, planned_slot_cap(p.slot_cap), 0, p.sp, qouts);
  jg.status = jq.status = status;
  {
    KScope k(K_DYPASS, st);
    const qlora_status s = cuda_status(launch_dypass(mt, mu, mb, jg, jq, (int)nch, status, st));
    if (s != QLORA_OK) return s;
  }
  const ReduceJob both[2] = {jg, jq};
  return reduce_now_or_later(both, 2, batch, st);
}

// One reduction output: columns [col0, col0 + width) of the partials, scaled, bf16
// into p (row stride ld, or transposed).
ReduceOut rout(bf16* p, int col0, int width, int ld, int transpose, float scale) {
  return {p, col0, width, ld, transpose, scale};
}
ReduceOuts routs(ReduceOut a, ReduceOut b = {nullptr, 0, 0, 0, 0, 0.f}, ReduceOut c = {nullptr, 0, 0, 0, 0, 0.f},
                 ReduceOut d = {nullptr, 0, 0, 0, 0, 0.f}) {
  ReduceOuts o;
  o.o[0] = a;
  o.o[1] = b;
  o.o[2] = c;
  o.o[3] = d;
  return o;
}

// NF4 weight maps for the GEMM B operand (K-major for forward, MN-major for dX);
// boxes follow the number of B columns each CTA dequantises (bnc).
bool map_nf4(CUtensorMap* codes, CUtensorMap* absmax, const Wt& w, bool bwd, int bnc) {
  const int64_t N = w.n_out, K = w.k_in;
  if (!bwd) {
    const int rows = bnc < 128 ? bnc : 128;
    return make_map(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.codes, K / 2, N, K / 2, 32, rows,
                    CU_TENSOR_MAP_SWIZZLE_32B) &&
           make_map(absmax, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, w.absmax, K / 64, N, K / 64, 4, rows,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  const int rb = bnc / 2;  // bytes of codes per W row per CTA tile
  const CUtensorMapSwizzle swz = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  return make_map(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.codes, K / 2, N, K / 2, rb, 64, swz) &&
         make_map(absmax, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, w.absmax, K / 64, N, K / 64, 4, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}
int lora_rows_box(int bnc) { return bnc < 128 ? bnc : 128; }

// Staged feed (tile configuration 4): the weight is dequantised once per call
// into a bf16 [N, K] buffer of the workspace and its B tiles arrive by TMA in
// the layout the in-mainloop dequantisers would have written.
bool is_staged(int tiles) { return tiles == 4; }
size_t stage_bytes(int64_t n_out, int64_t k_in) { return align256(static_cast<size_t>(n_out) * k_in * 2); }
bool map_staged(CUtensorMap* m, const void* wq, const Wt& w, bool bwd, int bnc) {
  const int64_t N = w.n_out, K = w.k_in;
  if (!bwd) return map_bf16(m, wq, K, N, K, 64, bnc < 128 ? bnc : 128, CU_TENSOR_MAP_SWIZZLE_128B);
  return map_bf16(m, wq, K, N, K, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Dequantises one weight (w1 == nullptr), two, or three (w2 too) in one launch into their staging buffers.
qlora_status stage_weights(const Wt& w0, bf16* dst0, const Wt* w1, bf16* dst1, cudaStream_t st,
                           const Wt* w2 = nullptr, bf16* dst2 = nullptr) {
  const Wt* w[3] = {&w0, w1, w2};
  bf16* const dst[3] = {dst0, dst1, dst2};
  const uint8_t* codes[3];
  const float* absmax[3];
  int64_t numel[3];
  bf16* out[3];
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (!w[i]) continue;
    codes[n] = w[i]->codes;
    absmax[n] = w[i]->absmax;
    numel[n] = w[i]->n_out * w[i]->k_in;
    out[n++] = dst[i];
  }
  KScope k(K_DEQUANT, st);
  return cuda_status(launch_nf4_dequantize(codes, absmax, numel, out, n, st, num_sms()));
}
// Output maps of the staged configuration's TMA-store epilogue: bf16 [rows, cols]
// with row stride ld, written in 32 x 32 boxes (64B swizzle).  No-ops otherwise.
bool map_outs(GemmMaps& maps, int tiles, int64_t rows, int64_t cols, int64_t ld, const void* o0,
              const void* o1 = nullptr, const void* o2 = nullptr) {
  if (!is_staged(tiles)) return true;
  const void* o[3] = {o0, o1, o2};
  for (int i = 0; i < 3; ++i)
    if (o[i] && !map_bf16(&maps.out[i], o[i], cols, rows, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return false;
  return true;
}
// B-operand maps of one weight (w1 == nullptr) or two (GEMM segments / gate-up halves 0 and 1) for
// either feed; under the staged feed NF4 weights are first dequantised into stage0 / stage1, and
// bf16 weights are read where they are (they always use the staged feed).
qlora_status map_weights(GemmMaps& maps, const Wt& w0, const Wt* w1, bool bwd, int tiles, bf16* stage0,
                         bf16* stage1, cudaStream_t st) {
  const int bnc = gemm_nf4_b_cols_per_cta(tiles);
  if (w0.w16) {
    if (!is_staged(tiles) || !map_staged(&maps.b[0], w0.w16, w0, bwd, bnc)) return QLORA_ERR_CUDA;
    if (w1 && !map_staged(&maps.b[1], w1->w16, *w1, bwd, bnc)) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  if (is_staged(tiles)) {
    const qlora_status s = stage_weights(w0, stage0, w1, stage1, st);
    if (s != QLORA_OK) return s;
    if (!map_staged(&maps.b[0], stage0, w0, bwd, bnc)) return QLORA_ERR_CUDA;
    if (w1 && !map_staged(&maps.b[1], stage1, *w1, bwd, bnc)) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  if (!map_nf4(&maps.codes[0], &maps.absmax[0], w0, bwd, bnc)) return QLORA_ERR_CUDA;
  if (w1 && !map_nf4(&maps.codes[1], &maps.absmax[1], *w1, bwd, bnc)) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// LoRA operand maps of the GEMM.  Left operand [rows, r] with row stride ld (s X A or
// s G); right factor: forward B [r, n], backward A [n, r].  The staged feed streams
// both as one 64-wide reduction block through the operand ring (zeros beyond the
// rank); the in-mainloop feed (rank 16) keeps its dedicated tiles.
bool map_lora_left(CUtensorMap* m, const void* p, int64_t rows, int r, int64_t ld, int tiles) {
  if (is_staged(tiles)) return map_bf16(m, p, r, rows, ld, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  return map_bf16(m, p, 16, rows, ld, 16, 128, CU_TENSOR_MAP_SWIZZLE_32B);
}
bool map_lora_right(CUtensorMap* m, const void* p, int64_t n, int r, bool bwd, int tiles) {
  const int bnc = gemm_nf4_b_cols_per_cta(tiles);
  if (is_staged(tiles)) {
    if (bwd) return map_bf16(m, p, r, n, r, 64, lora_rows_box(bnc), CU_TENSOR_MAP_SWIZZLE_128B);
    return map_bf16(m, p, n, r, n, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (bwd) return map_bf16(m, p, 16, n, 16, 16, lora_rows_box(bnc), CU_TENSOR_MAP_SWIZZLE_32B);
  return map_bf16(m, p, n, 16, n, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
}
// LoRA ranks: 16, 32 or 64 with the staged feed (configuration 4 or a bf16 base),
// 16 with the feeds that dequantise in the mainloop.
bool rank_ok(int r, int tiles) { return is_staged(tiles) ? (r == 16 || r == 32 || r == 64) : r == 16; }

// Configuration used by the projection and Q/K/V calls: the one selected, or the staged
// feed under the automatic setting (it is as fast or faster at every size measured).
int linear_tiles() { return g_tiles != 0 ? g_tiles : 4; }
// Configuration used by the NF4 gated-MLP calls for M tokens, width d and rank r.
int mlp_tiles(int64_t M, int64_t d, int r) {
  if (g_tiles != 0) return g_tiles;
  return (M <= kAutoMainloopMaxM && r == 16 && d % 256 == 0) ? 2 : 4;
}

qlora_status check_linear(const Lin* lin, int tiles) {
  if (!lin || !lin->A || !lin->B) return QLORA_ERR_INVALID_ARG;
  if (lin->w.w16 ? false : (!lin->w.codes || !lin->w.absmax)) return QLORA_ERR_INVALID_ARG;
  if (lin->w.n_out <= 0 || lin->w.k_in <= 0) return QLORA_ERR_INVALID_ARG;
  if (!rank_ok(lin->r, tiles)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (lin->w.k_in % 64 || lin->w.n_out % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  // The feeds that dequantise in the GEMM mainloop load each weight row's
  // absmax values by TMA, whose row stride (k_in / 64 binary32 values) must be
  // a multiple of 16 bytes.
  if (!is_staged(tiles) && !lin->w.w16 && lin->w.k_in % 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (lin->w.k_in > kMaxDim || lin->w.n_out > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (misaligned(lin->w.codes) || misaligned(lin->w.absmax) || misaligned(lin->w.w16) || misaligned(lin->A) ||
      misaligned(lin->B))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Y-side GEMM launch helpers -------------------------------------------------
qlora_status gemm_fwd(const Lin& lin, const bf16* X, int64_t M, const bf16* XAs, bf16* Y, int* status,
                      int tiles, bf16* stage, cudaStream_t st) {
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int64_t K = lin.w.k_in, N = lin.w.n_out;
  if (!map_bf16(&maps.a[0], X, K, M, K, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  const qlora_status s = map_weights(maps, lin.w, nullptr, false, tiles, stage, nullptr, st);
  if (s != QLORA_OK) return s;
  if (!map_lora_left(&maps.la[0], XAs, M, lin.r, lin.r, tiles)) return QLORA_ERR_CUDA;
  if (!map_lora_right(&maps.lb[0], lin.B, N, lin.r, false, tiles)) return QLORA_ERR_CUDA;
  maps.a[1] = maps.a[0];
  maps.codes[1] = maps.codes[0];
  maps.absmax[1] = maps.absmax[0];
  maps.b[1] = maps.b[0];
  maps.la[1] = maps.la[0];
  maps.lb[1] = maps.lb[0];
  if (!map_outs(maps, tiles, M, N, N, Y)) return QLORA_ERR_CUDA;
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.N = (int)N;
  a.nkb0 = (int)(K / 64);
  a.nkb1 = 0;
  a.lora = 1;
  a.lora_k16 = lin.r / 16;
  a.ldo = (int)N;
  a.D = Y;
  a.status = status;
  a.group_m = kGroupM;
  KScope k(K_GEMM_FWD, st);
  return cuda_status(launch_gemm_nf4(MODE_FWD, EPI_STORE, tiles, maps, a, st));
}

}  // namespace

// =========================================================== C entry points
extern "C" {

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "QLORA_ERR_UNSUPPORTED_SHAPE";
    case QLORA_ERR_MISALIGNED: return "QLORA_ERR_MISALIGNED";
    case QLORA_ERR_WORKSPACE_TOO_SMALL: return "QLORA_ERR_WORKSPACE_TOO_SMALL";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT";
    case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE";
  }
  return "QLORA_UNKNOWN_STATUS";
}

qlora_status qlora_nf4_codebook(float out[16]) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < 16; ++i) std::memcpy(&out[i], &h_nf4_bits[i], 4);
  return QLORA_OK;
}

int32_t qlora_checked_build(void) { return kChecked ? 1 : 0; }

qlora_status qlora_test_shrink_next_slot_cap(void) {
  g_shrink_slot_cap = 1;
  return QLORA_OK;
}

int32_t qlora_test_set_grid_cap(int32_t max_ctas) {
  const int32_t prev = g_grid_cap;
  if (max_ctas >= 0) g_grid_cap = max_ctas;
  return prev;
}

int32_t qlora_mlp_tile_config(int64_t M, int64_t d, int64_t h, int32_t r) {
  (void)h;
  return mlp_tiles(M, d, r);
}

int32_t qlora_set_tile_config(int32_t tiles) {
  const int32_t prev = g_tiles;
  if (tiles >= 0 && tiles <= 4) g_tiles = tiles;
  return prev;
}

qlora_status nf4_quantize(const qlora_bf16* w, int64_t n_out, int64_t k_in, uint8_t* codes, float* absmax,
                          qlora_stream_t stream) {
  if (n_out < 0 || k_in < 0) return QLORA_ERR_INVALID_ARG;
  if (k_in % 64) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (n_out == 0 || k_in == 0) return QLORA_OK;
  if (!w || !codes || !absmax) return QLORA_ERR_INVALID_ARG;
  if (misaligned(w) || misaligned(codes) || misaligned(absmax)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  KScope k(K_QUANT, st);
  return cuda_status(launch_nf4_quantize(reinterpret_cast<const bf16*>(w), n_out * k_in, codes, absmax, st));
}

qlora_status nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t n_out, int64_t k_in, qlora_bf16* out,
                            qlora_stream_t stream) {
  if (n_out < 0 || k_in < 0) return QLORA_ERR_INVALID_ARG;
  if (k_in % 64) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (n_out == 0 || k_in == 0) return QLORA_OK;
  if (!codes || !absmax || !out) return QLORA_ERR_INVALID_ARG;
  if (misaligned(codes) || misaligned(absmax) || misaligned(out)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  KScope k(K_DEQUANT, st);
  const int64_t numel = n_out * k_in;
  bf16* dst = reinterpret_cast<bf16*>(out);
  return cuda_status(launch_nf4_dequantize(&codes, &absmax, &numel, &dst, 1, st, num_sms()));
}

namespace {
// Linear workspace: [status word | 256 B][M x r vector][partials][staged weight, if `stage`]
size_t linear_ws(int64_t M, int64_t K, int64_t N, int r, bool stage) {
  const size_t vec = align256(static_cast<size_t>(M) * r * 2);
  size_t part = rowproj_part_bytes(M, K, r);
  part = std::max(part, dypass_part_bytes(M, N, r));
  part = std::max(part, colproj_part_bytes(M, K, r));
  return 256 + vec + align256(part) + (stage ? stage_bytes(N, K) : 0);
}
}  // namespace

size_t qlora_linear_workspace_bytes(int64_t M, int64_t K, int64_t N, int32_t r) {
  const int tiles = linear_tiles();
  if (M <= 0 || K <= 0 || N <= 0 || !rank_ok(r, tiles)) return 256;
  return linear_ws(M, K, N, r, is_staged(tiles));
}

namespace {
struct LinearWs {
  int* status;
  bf16* vec;
  float* part;
  bf16* stage;
};
LinearWs carve_linear(void* ws, int64_t M, int64_t K, int64_t N, int r, bool stage) {
  char* w = static_cast<char*>(ws);
  LinearWs l;
  l.status = reinterpret_cast<int*>(w);
  l.vec = reinterpret_cast<bf16*>(w + 256);
  l.part = reinterpret_cast<float*>(w + 256 + align256(static_cast<size_t>(M) * r * 2));
  l.stage = stage ? reinterpret_cast<bf16*>(w + linear_ws(M, K, N, r, true) - stage_bytes(N, K)) : nullptr;
  return l;
}
}  // namespace

static qlora_status linear_fwd(const Lin* lin, int tiles, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                               qlora_bf16* XA_saved, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_linear(lin, tiles);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;
  if (!X || !Y || !XA_saved || !ws) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(Y) || misaligned(XA_saved) || misaligned(ws)) return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t K = lin->w.k_in, N = lin->w.n_out;
  const int r = lin->r;
  const bool stage = is_staged(tiles) && !lin->w.w16;
  if (ws_bytes < linear_ws(M, K, N, r, stage)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LinearWs l = carve_linear(ws, M, K, N, r, stage);
  bf16* xa = reinterpret_cast<bf16*>(XA_saved);
  const bool scaled = lin->scale != 1.0f;
  bf16* XAs = scaled ? l.vec : xa;
  s = pass_rowproj(reinterpret_cast<const bf16*>(X), M, K, reinterpret_cast<const bf16*>(lin->A), nullptr, r, l.part,
                   routs(rout(xa, 0, r, r, 0, 1.f), rout(scaled ? XAs : nullptr, 0, r, r, 0, lin->scale)),
                   l.status, st);
  if (s != QLORA_OK) return s;
  return gemm_fwd(*lin, reinterpret_cast<const bf16*>(X), M, XAs, reinterpret_cast<bf16*>(Y), l.status, tiles,
                  l.stage, st);
}

static qlora_status linear_bwd(const Lin* lin, int tiles, const qlora_bf16* X, const qlora_bf16* XA_saved,
                        const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB, void* ws,
                        size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_linear(lin, tiles);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) {
    qlora_bf16* g[2] = {dA, dB};
    const int64_t n[2] = {lin->w.k_in * lin->r, lin->w.n_out * lin->r};
    return zero_adapter_grads(g, n, 2, reinterpret_cast<cudaStream_t>(stream));
  }
  if (!X || !XA_saved || !dY || !dX || !dA || !dB || !ws) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(XA_saved) || misaligned(dY) || misaligned(dX) || misaligned(dA) ||
      misaligned(dB) || misaligned(ws))
    return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t K = lin->w.k_in, N = lin->w.n_out;
  const int r = lin->r;
  const bool stage_w = is_staged(tiles) && !lin->w.w16;
  if (ws_bytes < linear_ws(M, K, N, r, stage_w)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LinearWs l = carve_linear(ws, M, K, N, r, stage_w);
  int* status = l.status;
  bf16* sG = l.vec;
  bf16* stage = l.stage;
  float* part = l.part;
  const float sc = lin->scale;
  // G = dY B^T (stored scaled: sG), dB = s (XA)^T dY
  s = pass_dypass(reinterpret_cast<const bf16*>(dY), M, N, reinterpret_cast<const bf16*>(XA_saved),
                  reinterpret_cast<const bf16*>(lin->B), r, part, routs(rout(sG, 0, r, r, 0, sc)),
                  routs(rout(reinterpret_cast<bf16*>(dB), 0, r, (int)N, 1, sc)), status, st);
  if (s != QLORA_OK) return s;
  // dX = dY W + (s G) A^T
  {
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!map_bf16(&maps.a[0], dY, N, M, N, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    if ((s = map_weights(maps, lin->w, nullptr, true, tiles, stage, nullptr, st)) != QLORA_OK) return s;
    if (!map_lora_left(&maps.la[0], sG, M, r, r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[0], lin->A, K, r, true, tiles)) return QLORA_ERR_CUDA;
    maps.a[1] = maps.a[0];
    maps.codes[1] = maps.codes[0];
    maps.absmax[1] = maps.absmax[0];
    maps.b[1] = maps.b[0];
    maps.la[1] = maps.la[0];
    maps.lb[1] = maps.lb[0];
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = (int)M;
    a.N = (int)K;
    a.nkb0 = (int)cdiv(N, 64);
    a.lora = 1;
    a.lora_k16 = r / 16;
    a.ldo = (int)K;
    a.D = reinterpret_cast<bf16*>(dX);
    if (!map_outs(maps, tiles, M, K, K, dX)) return QLORA_ERR_CUDA;
    a.status = status;
    a.group_m = kGroupM;
    KScope k(K_GEMM_BWD, st);
    s = cuda_status(launch_gemm_nf4(MODE_BWD, EPI_STORE, tiles, maps, a, st));
    if (s != QLORA_OK) return s;
  }
  // dA = X^T (s G)
  return pass_colproj(reinterpret_cast<const bf16*>(X), M, K, sG, r, part,
                      routs(rout(reinterpret_cast<bf16*>(dA), 0, r, r, 0, 1.f)), status, st);
}

namespace {
// The backward reduces the dA_d pass and the two passes over dE and dG in one
// launch, so their partials sit side by side: [dA_d | dE pass | dG pass].
size_t mlp_bwd_part_dad(int64_t M, int64_t h, int r) { return align256(colproj_part_bytes(M, h, r)); }
size_t mlp_bwd_part_dy(int64_t M, int64_t h, int r) { return align256(dypass_part_bytes(M, h, r)); }
// MLP workspace: [status | 256 B][dE][dG][5 rank vectors][partials][two staged weights, if `stage`]
size_t mlp_ws(int64_t M, int64_t d, int64_t h, int r, bool stage) {
  const size_t big = align256(static_cast<size_t>(M) * h * 2);
  const size_t vec = align256(static_cast<size_t>(M) * r * 2);
  size_t part = rowproj_part_bytes(M, d, 2 * r);
  part = std::max(part, rowproj_part_bytes(M, h, r));
  part = std::max(part, dypass_part_bytes(M, d, r));
  part = std::max(part, mlp_bwd_part_dad(M, h, r) + 2 * mlp_bwd_part_dy(M, h, r));
  part = std::max(part, colproj_part_bytes(M, d, 2 * r));
  return 256 + 2 * big + 5 * vec + align256(part) + (stage ? 2 * stage_bytes(h, d) : 0);
}
}  // namespace

size_t qlora_mlp_workspace_bytes(int64_t M, int64_t d, int64_t h, int32_t r) {
  const int tiles = mlp_tiles(M, d, r);
  if (M <= 0 || d <= 0 || h <= 0 || !rank_ok(r, tiles)) return 256;
  return mlp_ws(M, d, h, r, is_staged(tiles));
}

namespace {
struct MlpWs {
  int* status;
  bf16 *dE, *dG, *v0, *v1, *v2, *gu;  // v*: [M, r] vectors; gu: [M, 2r]
  float* part;
  bf16 *stage0, *stage1;  // staged feed: room for two dequantised [h, d] weights (gate, up; or down)
};
MlpWs carve_mlp(void* ws, int64_t M, int64_t d, int64_t h, int r, bool stage) {
  char* w = static_cast<char*>(ws);
  const size_t big = align256(static_cast<size_t>(M) * h * 2);
  const size_t vec = align256(static_cast<size_t>(M) * r * 2);
  MlpWs m;
  m.status = reinterpret_cast<int*>(w);
  size_t off = 256;
  m.dE = reinterpret_cast<bf16*>(w + off); off += big;
  m.dG = reinterpret_cast<bf16*>(w + off); off += big;
  m.v0 = reinterpret_cast<bf16*>(w + off); off += vec;
  m.v1 = reinterpret_cast<bf16*>(w + off); off += vec;
  m.v2 = reinterpret_cast<bf16*>(w + off); off += vec;
  m.gu = reinterpret_cast<bf16*>(w + off); off += 2 * vec;
  m.part = reinterpret_cast<float*>(w + off);
  const size_t total = mlp_ws(M, d, h, r, true);
  m.stage0 = m.stage1 = nullptr;
  if (stage) {
    m.stage0 = reinterpret_cast<bf16*>(w + total - 2 * stage_bytes(h, d));
    m.stage1 = reinterpret_cast<bf16*>(w + total - stage_bytes(h, d));
  }
  return m;
}
qlora_status check_mlp(const Lin* g, const Lin* u, const Lin* d, int tiles) {
  qlora_status s;
  if ((s = check_linear(g, tiles)) != QLORA_OK || (s = check_linear(u, tiles)) != QLORA_OK ||
      (s = check_linear(d, tiles)) != QLORA_OK)
    return s;
  if (g->r != u->r || g->r != d->r) return QLORA_ERR_UNSUPPORTED_SHAPE;  // one rank for the three
  if (g->w.n_out != u->w.n_out || g->w.k_in != u->w.k_in || d->w.k_in != g->w.n_out || d->w.n_out != g->w.k_in)
    return QLORA_ERR_INVALID_ARG;
  if (g->w.n_out % 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!g->w.w16 != !u->w.w16 || !g->w.w16 != !d->w.w16) return QLORA_ERR_INVALID_ARG;  // one base format
  return QLORA_OK;
}
}  // namespace

static qlora_status mlp_fwd(qlora_act act, const Lin* gate, const Lin* up, const Lin* down, int tiles, const qlora_bf16* X,
                     int64_t M, qlora_bf16* Y, const qlora_mlp_saved* sv, void* ws, size_t ws_bytes,
                     qlora_stream_t stream) {
  if (act != QLORA_ACT_SWIGLU && act != QLORA_ACT_GEGLU_TANH) return QLORA_ERR_INVALID_ARG;
  qlora_status s = check_mlp(gate, up, down, tiles);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;
  if (!X || !Y || !sv || !sv->E || !sv->G || !sv->H || !sv->XA_g || !sv->XA_u || !sv->HA_d || !ws)
    return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(Y) || misaligned(sv->E) || misaligned(sv->G) || misaligned(sv->H) ||
      misaligned(sv->XA_g) || misaligned(sv->XA_u) || misaligned(sv->HA_d) || misaligned(ws))
    return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t d = gate->w.k_in, h = gate->w.n_out;
  const int r = gate->r;
  const bool stage = is_staged(tiles) && !gate->w.w16;
  if (ws_bytes < mlp_ws(M, d, h, r, stage)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  MlpWs w = carve_mlp(ws, M, d, h, r, stage);
  const bf16* x = reinterpret_cast<const bf16*>(X);
  bf16* xag = reinterpret_cast<bf16*>(sv->XA_g);
  bf16* xau = reinterpret_cast<bf16*>(sv->XA_u);
  bf16* had = reinterpret_cast<bf16*>(sv->HA_d);
  bf16* xags = gate->scale != 1.f ? w.v0 : xag;
  bf16* xaus = up->scale != 1.f ? w.v1 : xau;
  bf16* hads = down->scale != 1.f ? w.v2 : had;
  // XA_g, XA_u = X [A_g | A_u] (one pass over X)
  s = pass_rowproj(x, M, d, reinterpret_cast<const bf16*>(gate->A), reinterpret_cast<const bf16*>(up->A), r, w.part,
                   routs(rout(xag, 0, r, r, 0, 1.f), rout(xau, r, r, r, 0, 1.f),
                         rout(xags != xag ? xags : nullptr, 0, r, r, 0, gate->scale),
                         rout(xaus != xau ? xaus : nullptr, r, r, r, 0, up->scale)),
                   w.status, st);
  if (s != QLORA_OK) return s;
  // gate/up GEMM with the gated activation in the epilogue -> E, G, H
  {
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!map_bf16(&maps.a[0], x, d, M, d, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    maps.a[1] = maps.a[0];
    if ((s = map_weights(maps, gate->w, &up->w, false, tiles, w.stage0, w.stage1, st)) != QLORA_OK) return s;
    if (!map_lora_left(&maps.la[0], xags, M, r, r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_left(&maps.la[1], xaus, M, r, r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[0], gate->B, h, r, false, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[1], up->B, h, r, false, tiles)) return QLORA_ERR_CUDA;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = (int)M;
    a.N = (int)h;
    a.nkb0 = (int)(d / 64);
    a.lora = 2;
    a.lora_k16 = r / 16;
    a.act = act == QLORA_ACT_SWIGLU ? ACT_SILU : ACT_GELU_TANH;
    a.ldo = (int)h;
    a.E = reinterpret_cast<bf16*>(sv->E);
    a.G = reinterpret_cast<bf16*>(sv->G);
    a.H = reinterpret_cast<bf16*>(sv->H);
    if (!map_outs(maps, tiles, M, h, h, sv->E, sv->G, sv->H)) return QLORA_ERR_CUDA;
    a.status = w.status;
    a.group_m = kGroupM;
    KScope k(K_GEMM_GLU_FWD, st);
    s = cuda_status(launch_gemm_nf4(MODE_FWD_GLU, EPI_GLU_FWD, tiles, maps, a, st));
    if (s != QLORA_OK) return s;
  }
  // HA_d = H A_d
  s = pass_rowproj(reinterpret_cast<const bf16*>(sv->H), M, h, reinterpret_cast<const bf16*>(down->A), nullptr, r,
                   w.part, routs(rout(had, 0, r, r, 0, 1.f), rout(hads != had ? hads : nullptr, 0, r, r, 0, down->scale)),
                   w.status, st);
  if (s != QLORA_OK) return s;
  // Y = H W_d^T + (s H A_d) B_d
  return gemm_fwd(*down, reinterpret_cast<const bf16*>(sv->H), M, hads, reinterpret_cast<bf16*>(Y), w.status, tiles,
                  w.stage0, st);
}

static qlora_status mlp_bwd(qlora_act act, const Lin* gate, const Lin* up, const Lin* down, int tiles, const qlora_bf16* X,
                     const qlora_mlp_saved* sv, const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g,
                     qlora_bf16* dB_g, qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d,
                     void* ws, size_t ws_bytes, qlora_stream_t stream, qlora_event_t early = nullptr) {
  if (act != QLORA_ACT_SWIGLU && act != QLORA_ACT_GEGLU_TANH) return QLORA_ERR_INVALID_ARG;
  qlora_status s = check_mlp(gate, up, down, tiles);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) {
    const int64_t dm = gate->w.k_in, hm = gate->w.n_out, rm = gate->r;
    qlora_bf16* g[6] = {dA_g, dB_g, dA_u, dB_u, dA_d, dB_d};
    const int64_t n[6] = {dm * rm, rm * hm, dm * rm, rm * hm, hm * rm, rm * dm};
    s = zero_adapter_grads(g, n, 6, reinterpret_cast<cudaStream_t>(stream));
    if (s == QLORA_OK && early &&
        cudaEventRecord(reinterpret_cast<cudaEvent_t>(early), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return s;
  }
  if (!X || !sv || !sv->E || !sv->G || !sv->H || !sv->XA_g || !sv->XA_u || !sv->HA_d || !dY || !dX || !dA_g ||
      !dB_g || !dA_u || !dB_u || !dA_d || !dB_d || !ws)
    return QLORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, sv->E, sv->G, sv->H, sv->XA_g, sv->XA_u, sv->HA_d, dY, dX, dA_g, dB_g, dA_u, dB_u, dA_d,
                        dB_d, ws};
  for (const void* p : ptrs)
    if (misaligned(p)) return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t d = gate->w.k_in, h = gate->w.n_out;
  const int r = gate->r;
  const bool stage = is_staged(tiles) && !gate->w.w16;
  if (ws_bytes < mlp_ws(M, d, h, r, stage)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  MlpWs w = carve_mlp(ws, M, d, h, r, stage);
  bf16* sGd = w.v0;
  // 1. G_d = dY B_d^T (scaled), dB_d = s_d HA_d^T dY
  s = pass_dypass(reinterpret_cast<const bf16*>(dY), M, d, reinterpret_cast<const bf16*>(sv->HA_d),
                  reinterpret_cast<const bf16*>(down->B), r, w.part, routs(rout(sGd, 0, r, r, 0, down->scale)),
                  routs(rout(reinterpret_cast<bf16*>(dB_d), 0, r, (int)d, 1, down->scale)), w.status, st);
  if (s != QLORA_OK) return s;
  // 2. dH = dY W_d + sG_d A_d^T, with dE, dG formed in the epilogue
  {
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!map_bf16(&maps.a[0], dY, d, M, d, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    if ((s = map_weights(maps, down->w, nullptr, true, tiles, w.stage0, nullptr, st)) != QLORA_OK) return s;
    if (!map_lora_left(&maps.la[0], sGd, M, r, r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[0], down->A, h, r, true, tiles)) return QLORA_ERR_CUDA;
    maps.a[1] = maps.a[0];
    maps.codes[1] = maps.codes[0];
    maps.absmax[1] = maps.absmax[0];
    maps.b[1] = maps.b[0];
    maps.la[1] = maps.la[0];
    maps.lb[1] = maps.lb[0];
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = (int)M;
    a.N = (int)h;
    a.nkb0 = (int)cdiv(d, 64);
    a.lora = 1;
    a.lora_k16 = r / 16;
    a.act = act == QLORA_ACT_SWIGLU ? ACT_SILU : ACT_GELU_TANH;
    a.ldo = (int)h;
    a.Ein = reinterpret_cast<const bf16*>(sv->E);
    a.Gin = reinterpret_cast<const bf16*>(sv->G);
    a.dE = w.dE;
    a.dG = w.dG;
    if (!map_outs(maps, tiles, M, h, h, w.dE, w.dG)) return QLORA_ERR_CUDA;
    a.status = w.status;
    a.group_m = kGroupM;
    KScope k(K_GEMM_GLU_BWD, st);
    s = cuda_status(launch_gemm_nf4(MODE_BWD, EPI_GLU_BWD, tiles, maps, a, st));
    if (s != QLORA_OK) return s;
  }
  // 3. dA_d = H^T (s_d G_d)
  // 4. G_g = dE B_g^T, dB_g = s_g XA_g^T dE ; G_u = dG B_u^T, dB_u = s_u XA_u^T dG
  // Nothing reads dA_d before the end of the call, so its partial sums are
  // reduced in one launch with those of the two passes of step 4.
  {
    ReduceBatch rb;
    float* part_dad = w.part;
    float* part_de = reinterpret_cast<float*>(reinterpret_cast<char*>(w.part) + mlp_bwd_part_dad(M, h, r));
    float* part_dg = reinterpret_cast<float*>(reinterpret_cast<char*>(part_de) + mlp_bwd_part_dy(M, h, r));
    s = pass_colproj(reinterpret_cast<const bf16*>(sv->H), M, h, sGd, r, part_dad,
                     routs(rout(reinterpret_cast<bf16*>(dA_d), 0, r, r, 0, 1.f)), w.status, st, 0, 0, &rb);
    if (s != QLORA_OK) return s;
    s = pass_dypass(w.dE, M, h, reinterpret_cast<const bf16*>(sv->XA_g), reinterpret_cast<const bf16*>(gate->B), r,
                    part_de, routs(rout(w.gu, 0, r, 2 * r, 0, gate->scale)),
                    routs(rout(reinterpret_cast<bf16*>(dB_g), 0, r, (int)h, 1, gate->scale)), w.status, st, 0, 0,
                    &rb);
    if (s != QLORA_OK) return s;
    s = pass_dypass(w.dG, M, h, reinterpret_cast<const bf16*>(sv->XA_u), reinterpret_cast<const bf16*>(up->B), r,
                    part_dg, routs(rout(w.gu + r, 0, r, 2 * r, 0, up->scale)),
                    routs(rout(reinterpret_cast<bf16*>(dB_u), 0, r, (int)h, 1, up->scale)), w.status, st, 0, 0,
                    &rb);
    if (s != QLORA_OK) return s;
    if ((s = flush_reduce(rb, st)) != QLORA_OK) return s;
  }
  // dA_d, dB_d, dB_g and dB_u are final: a data-parallel caller may start summing them across ranks
  if (early && cudaEventRecord(reinterpret_cast<cudaEvent_t>(early), st) != cudaSuccess) return QLORA_ERR_CUDA;
  // 5. dX = [dE | dG] [W_g ; W_u] + [sG_g | sG_u] [A_g^T ; A_u^T]
  {
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!map_bf16(&maps.a[0], w.dE, h, M, h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    if (!map_bf16(&maps.a[1], w.dG, h, M, h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    if ((s = map_weights(maps, gate->w, &up->w, true, tiles, w.stage0, w.stage1, st)) != QLORA_OK) return s;
    if (!map_lora_left(&maps.la[0], w.gu, M, r, 2 * r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_left(&maps.la[1], w.gu + r, M, r, 2 * r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[0], gate->A, d, r, true, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[1], up->A, d, r, true, tiles)) return QLORA_ERR_CUDA;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = (int)M;
    a.N = (int)d;
    a.nkb0 = (int)cdiv(h, 64);
    a.nkb1 = (int)cdiv(h, 64);
    a.lora = 2;
    a.lora_k16 = r / 16;
    a.ldo = (int)d;
    a.D = reinterpret_cast<bf16*>(dX);
    if (!map_outs(maps, tiles, M, d, d, dX)) return QLORA_ERR_CUDA;
    a.status = w.status;
    a.group_m = kGroupM;
    KScope k(K_GEMM_BWD, st);
    s = cuda_status(launch_gemm_nf4(MODE_BWD, EPI_STORE, tiles, maps, a, st));
    if (s != QLORA_OK) return s;
  }
  // 6. [dA_g | dA_u] = X^T [sG_g | sG_u]
  return pass_colproj(reinterpret_cast<const bf16*>(X), M, d, w.gu, 2 * r, w.part,
                      routs(rout(reinterpret_cast<bf16*>(dA_g), 0, r, r, 0, 1.f),
                            rout(reinterpret_cast<bf16*>(dA_u), r, r, r, 0, 1.f)),
                      w.status, st);
}

// ------------------------------------------------------------ fused QKV --
namespace {
// QKV workspace: [status | 256 B][s XA, M x 3r][s G, M x 3r][partials][staged [nq+nk+nv, K] weight]
// The backward's three dY passes (q, k, v) are reduced in one launch, so their
// partial sums sit side by side: [q pass | k pass | v pass].
size_t qkv_dy_part(int64_t M, int64_t n, int r) { return align256(dypass_part_bytes(M, n, r)); }
size_t qkv_ws(int64_t M, int64_t K, int64_t nq, int64_t nk, int64_t nv, int r) {
  const size_t vec = align256(static_cast<size_t>(M) * 3 * r * 2);
  size_t part = rowproj_part_bytes(M, K, 3 * r);
  part = std::max(part, qkv_dy_part(M, nq, r) + qkv_dy_part(M, nk, r) + qkv_dy_part(M, nv, r));
  part = std::max(part, 3 * r <= 128 ? colproj_part_bytes(M, K, 3 * r) : colproj_part_bytes(M, K, r));
  return 256 + 2 * vec + align256(part) + stage_bytes(nq + nk + nv, K);
}
qlora_status check_qkv(const Lin* q, const Lin* k, const Lin* v) {
  qlora_status s;
  for (const Lin* l : {q, k, v})
    if ((s = check_linear(l, 4)) != QLORA_OK) return s;
  if (q->w.k_in != k->w.k_in || q->w.k_in != v->w.k_in) return QLORA_ERR_INVALID_ARG;
  if (q->r != k->r || q->r != v->r) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (q->w.n_out % 256 || k->w.n_out % 256) return QLORA_ERR_UNSUPPORTED_SHAPE;  // tiles never straddle
  if (q->w.w16 || k->w.w16 || v->w.w16) return QLORA_ERR_INVALID_ARG;
  if (q->w.n_out + k->w.n_out + v->w.n_out > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}
// the three weights dequantised (one launch) into consecutive rows of one [nq + nk + nv, K] buffer
qlora_status stage_qkv(const Lin* q, const Lin* k, const Lin* v, bf16* stage, cudaStream_t st) {
  const int64_t K = q->w.k_in;
  return stage_weights(q->w, stage, &k->w, stage + q->w.n_out * K, st, &v->w,
                       stage + (q->w.n_out + k->w.n_out) * K);
}
}  // namespace

size_t qlora_qkv_workspace_bytes(int64_t M, int64_t k_in, int64_t nq, int64_t nk, int64_t nv, int32_t r) {
  if (M <= 0 || k_in <= 0 || nq <= 0 || nk <= 0 || nv <= 0 || !rank_ok(r, 4)) return 256;
  return qkv_ws(M, k_in, nq, nk, nv, r);
}

qlora_status qlora_qkv_fwd(const qlora_lora_linear* q_, const qlora_lora_linear* k_, const qlora_lora_linear* v_,
                           const qlora_bf16* X, int64_t M, qlora_bf16* Y, qlora_bf16* XA_saved, void* ws,
                           size_t ws_bytes, qlora_stream_t stream) {
  if (!q_ || !k_ || !v_) return QLORA_ERR_INVALID_ARG;
  const Lin lq = lin_of(*q_), lk = lin_of(*k_), lv = lin_of(*v_);
  const Lin* L[3] = {&lq, &lk, &lv};
  qlora_status s = check_qkv(&lq, &lk, &lv);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;
  if (!X || !Y || !XA_saved || !ws) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(Y) || misaligned(XA_saved) || misaligned(ws)) return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int r = lq.r;
  const int64_t K = lq.w.k_in, nq = lq.w.n_out, nk = lk.w.n_out, nv = lv.w.n_out, Nt = nq + nk + nv;
  if (ws_bytes < qkv_ws(M, K, nq, nk, nv, r)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const size_t vec = align256(static_cast<size_t>(M) * 3 * r * 2);
  int* status = reinterpret_cast<int*>(w);
  bf16* sxa = reinterpret_cast<bf16*>(w + 256);
  float* part = reinterpret_cast<float*>(w + 256 + 2 * vec);
  bf16* stage = reinterpret_cast<bf16*>(w + qkv_ws(M, K, nq, nk, nv, r) - stage_bytes(Nt, K));
  bf16* xa = reinterpret_cast<bf16*>(XA_saved);
  // [XA_q | XA_k | XA_v] = X [A_q | A_k | A_v] in one pass over X, plus the s-scaled copies
  s = pass_rowproj(reinterpret_cast<const bf16*>(X), M, K, reinterpret_cast<const bf16*>(lq.A),
                   reinterpret_cast<const bf16*>(lk.A), r, part,
                   routs(rout(xa, 0, 3 * r, 3 * r, 0, 1.f), rout(sxa, 0, r, 3 * r, 0, lq.scale),
                         rout(sxa + r, r, r, 3 * r, 0, lk.scale), rout(sxa + 2 * r, 2 * r, r, 3 * r, 0, lv.scale)),
                   status, st, reinterpret_cast<const bf16*>(lv.A));
  if (s != QLORA_OK) return s;
  if ((s = stage_qkv(&lq, &lk, &lv, stage, st)) != QLORA_OK) return s;
  // Y = X [W_q ; W_k ; W_v]^T + per column block s_p (X A_p) B_p
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const Wt wall = {nullptr, nullptr, nullptr, Nt, K};
  const int tiles = 4;
  if (!map_bf16(&maps.a[0], X, K, M, K, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
  if (!map_staged(&maps.b[0], stage, wall, false, gemm_nf4_b_cols_per_cta(tiles))) return QLORA_ERR_CUDA;
  for (int p = 0; p < 3; ++p) {
    if (!map_lora_left(&maps.la[p], sxa + p * r, M, r, 3 * r, tiles)) return QLORA_ERR_CUDA;
    if (!map_lora_right(&maps.lb[p], L[p]->B, L[p]->w.n_out, r, false, tiles)) return QLORA_ERR_CUDA;
  }
  maps.a[1] = maps.a[0];
  maps.b[1] = maps.b[0];
  if (!map_outs(maps, tiles, M, Nt, Nt, Y)) return QLORA_ERR_CUDA;
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.N = (int)Nt;
  a.nkb0 = (int)(K / 64);
  a.lora = 1;
  a.lora_k16 = r / 16;
  a.ncut[0] = (int)nq;
  a.ncut[1] = (int)(nq + nk);
  a.ldo = (int)Nt;
  a.D = reinterpret_cast<bf16*>(Y);
  a.status = status;
  a.group_m = kGroupM;
  KScope kk(K_GEMM_FWD, st);
  return cuda_status(launch_gemm_nf4(MODE_FWD, EPI_STORE, tiles, maps, a, st));
}

qlora_status qlora_qkv_bwd(const qlora_lora_linear* q_, const qlora_lora_linear* k_, const qlora_lora_linear* v_,
                           const qlora_bf16* X, const qlora_bf16* XA_saved, const qlora_bf16* dY, int64_t M,
                           qlora_bf16* dX, qlora_bf16* dA_q, qlora_bf16* dB_q, qlora_bf16* dA_k, qlora_bf16* dB_k,
                           qlora_bf16* dA_v, qlora_bf16* dB_v, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!q_ || !k_ || !v_) return QLORA_ERR_INVALID_ARG;
  const Lin lq = lin_of(*q_), lk = lin_of(*k_), lv = lin_of(*v_);
  const Lin* L[3] = {&lq, &lk, &lv};
  qlora_status s = check_qkv(&lq, &lk, &lv);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  qlora_bf16* dA[3] = {dA_q, dA_k, dA_v};
  qlora_bf16* dB[3] = {dB_q, dB_k, dB_v};
  if (M == 0) {
    qlora_bf16* g[6] = {dA_q, dB_q, dA_k, dB_k, dA_v, dB_v};
    int64_t n[6];
    for (int p = 0; p < 3; ++p) {
      n[2 * p] = L[p]->w.k_in * L[p]->r;       // dA [K, r]
      n[2 * p + 1] = L[p]->r * L[p]->w.n_out;  // dB [r, n_p]
    }
    return zero_adapter_grads(g, n, 6, reinterpret_cast<cudaStream_t>(stream));
  }
  if (!X || !XA_saved || !dY || !dX || !ws) return QLORA_ERR_INVALID_ARG;
  for (int p = 0; p < 3; ++p)
    if (!dA[p] || !dB[p]) return QLORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, XA_saved, dY, dX, dA_q, dB_q, dA_k, dB_k, dA_v, dB_v, ws};
  for (const void* p : ptrs)
    if (misaligned(p)) return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int r = lq.r;
  const int64_t K = lq.w.k_in, nq = lq.w.n_out, nk = lk.w.n_out, nv = lv.w.n_out, Nt = nq + nk + nv;
  const int64_t off[3] = {0, nq, nq + nk};
  if (ws_bytes < qkv_ws(M, K, nq, nk, nv, r)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const size_t vec = align256(static_cast<size_t>(M) * 3 * r * 2);
  int* status = reinterpret_cast<int*>(w);
  bf16* sg = reinterpret_cast<bf16*>(w + 256 + vec);
  float* part = reinterpret_cast<float*>(w + 256 + 2 * vec);
  bf16* stage = reinterpret_cast<bf16*>(w + qkv_ws(M, K, nq, nk, nv, r) - stage_bytes(Nt, K));
  const bf16* dy = reinterpret_cast<const bf16*>(dY);
  const bf16* xa = reinterpret_cast<const bf16*>(XA_saved);
  // per projection: G_p = dY_p B_p^T (stored s_p-scaled into [sG_q | sG_k | sG_v]), dB_p = s_p XA_p^T dY_p;
  // the three passes' reductions share one launch (each pass has its own partial region)
  {
    ReduceBatch rb;
    char* pp = reinterpret_cast<char*>(part);
    for (int p = 0; p < 3; ++p) {
      s = pass_dypass(dy + off[p], M, L[p]->w.n_out, xa + p * r, reinterpret_cast<const bf16*>(L[p]->B), r,
                      reinterpret_cast<float*>(pp), routs(rout(sg + p * r, 0, r, 3 * r, 0, L[p]->scale)),
                      routs(rout(reinterpret_cast<bf16*>(dB[p]), 0, r, (int)L[p]->w.n_out, 1, L[p]->scale)), status,
                      st, Nt, 3 * r, &rb);
      if (s != QLORA_OK) return s;
      pp += qkv_dy_part(M, L[p]->w.n_out, r);
    }
    if ((s = flush_reduce(rb, st)) != QLORA_OK) return s;
  }
  if ((s = stage_qkv(&lq, &lk, &lv, stage, st)) != QLORA_OK) return s;
  // dX = dY [W_q ; W_k ; W_v] + sum_p (s_p G_p) A_p^T: one concatenated reduction and three LoRA blocks
  {
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const Wt wall = {nullptr, nullptr, nullptr, Nt, K};
    const int tiles = 4;
    if (!map_bf16(&maps.a[0], dY, Nt, M, Nt, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    if (!map_staged(&maps.b[0], stage, wall, true, gemm_nf4_b_cols_per_cta(tiles))) return QLORA_ERR_CUDA;
    for (int p = 0; p < 3; ++p) {
      if (!map_lora_left(&maps.la[p], sg + p * r, M, r, 3 * r, tiles)) return QLORA_ERR_CUDA;
      if (!map_lora_right(&maps.lb[p], L[p]->A, K, r, true, tiles)) return QLORA_ERR_CUDA;
    }
    maps.a[1] = maps.a[0];
    maps.b[1] = maps.b[0];
    if (!map_outs(maps, tiles, M, K, K, dX)) return QLORA_ERR_CUDA;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = (int)M;
    a.N = (int)K;
    a.nkb0 = (int)cdiv(Nt, 64);
    a.lora = 3;
    a.lora_k16 = r / 16;
    a.ldo = (int)K;
    a.D = reinterpret_cast<bf16*>(dX);
    a.status = status;
    a.group_m = kGroupM;
    KScope kk(K_GEMM_BWD, st);
    s = cuda_status(launch_gemm_nf4(MODE_BWD, EPI_STORE, tiles, maps, a, st));
    if (s != QLORA_OK) return s;
  }
  // dA_p = X^T (s_p G_p): one pass over X while 3r fits a factor tile
  const bf16* x = reinterpret_cast<const bf16*>(X);
  if (3 * r <= 128)
    return pass_colproj(x, M, K, sg, 3 * r, part,
                        routs(rout(reinterpret_cast<bf16*>(dA_q), 0, r, r, 0, 1.f),
                              rout(reinterpret_cast<bf16*>(dA_k), r, r, r, 0, 1.f),
                              rout(reinterpret_cast<bf16*>(dA_v), 2 * r, r, r, 0, 1.f)),
                        status, st);
  for (int p = 0; p < 3; ++p) {
    s = pass_colproj(x, M, K, sg + p * r, r, part, routs(rout(reinterpret_cast<bf16*>(dA[p]), 0, r, r, 0, 1.f)),
                     status, st, 0, 3 * r);
    if (s != QLORA_OK) return s;
  }
  return QLORA_OK;
}

// ---------------------------------------------------------------- norm ----
qlora_status qlora_rmsnorm_fwd(const qlora_bf16* X, const qlora_bf16* w, int64_t M, int64_t d, float eps,
                               int32_t plus_one, qlora_bf16* Y, float* rstd, qlora_stream_t stream) {
  if (M < 0 || d <= 0 || !(eps >= 0.f)) return QLORA_ERR_INVALID_ARG;
  if (d % 8 || d > (1 << 30) || M > (1 << 30)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return QLORA_OK;
  if (!X || !w || !Y || !rstd) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(w) || misaligned(Y) || misaligned(rstd)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  KScope k(K_NORM_FWD, st);
  return cuda_status(launch_rmsnorm_fwd(reinterpret_cast<const bf16*>(X), reinterpret_cast<const bf16*>(w), (int)M,
                                        (int)d, eps, plus_one ? 1 : 0, reinterpret_cast<bf16*>(Y), rstd, st));
}

qlora_status qlora_rmsnorm_bwd(const qlora_bf16* X, const qlora_bf16* w, const float* rstd, const qlora_bf16* dY,
                               int64_t M, int64_t d, int32_t plus_one, qlora_bf16* dX, qlora_stream_t stream) {
  if (M < 0 || d <= 0) return QLORA_ERR_INVALID_ARG;
  if (d % 8 || d > (1 << 30) || M > (1 << 30)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return QLORA_OK;
  if (!X || !w || !rstd || !dY || !dX) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(w) || misaligned(rstd) || misaligned(dY) || misaligned(dX))
    return QLORA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  KScope k(K_NORM_BWD, st);
  return cuda_status(launch_rmsnorm_bwd(reinterpret_cast<const bf16*>(X), reinterpret_cast<const bf16*>(w), rstd,
                                        reinterpret_cast<const bf16*>(dY), (int)M, (int)d, plus_one ? 1 : 0,
                                        reinterpret_cast<bf16*>(dX), st));
}

// NF4 entry points: the current tile configuration.
qlora_status qlora_linear_fwd(const qlora_lora_linear* lin, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                              qlora_bf16* XA_saved, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!lin) return QLORA_ERR_INVALID_ARG;
  const Lin l = lin_of(*lin);
  return linear_fwd(&l, linear_tiles(), X, M, Y, XA_saved, ws, ws_bytes, stream);
}
qlora_status qlora_linear_bwd(const qlora_lora_linear* lin, const qlora_bf16* X, const qlora_bf16* XA_saved,
                              const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB,
                              void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!lin) return QLORA_ERR_INVALID_ARG;
  const Lin l = lin_of(*lin);
  return linear_bwd(&l, linear_tiles(), X, XA_saved, dY, M, dX, dA, dB, ws, ws_bytes, stream);
}
qlora_status qlora_mlp_fwd(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                           const qlora_lora_linear* down, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                           const qlora_mlp_saved* sv, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!gate || !up || !down) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_fwd(act, &g, &u, &d, mlp_tiles(M, g.w.k_in, g.r), X, M, Y, sv, ws, ws_bytes, stream);
}
qlora_status qlora_mlp_bwd(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                           const qlora_lora_linear* down, const qlora_bf16* X, const qlora_mlp_saved* sv,
                           const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                           qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d, void* ws,
                           size_t ws_bytes, qlora_stream_t stream) {
  if (!gate || !up || !down) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_bwd(act, &g, &u, &d, mlp_tiles(M, g.w.k_in, g.r), X, sv, dY, M, dX, dA_g, dB_g, dA_u, dB_u, dA_d, dB_d,
                 ws, ws_bytes,
                 stream);
}

qlora_status qlora_mlp_bwd_ev(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                              const qlora_lora_linear* down, const qlora_bf16* X, const qlora_mlp_saved* sv,
                              const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                              qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d, void* ws,
                              size_t ws_bytes, qlora_stream_t stream, qlora_event_t early_grads) {
  if (!gate || !up || !down) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_bwd(act, &g, &u, &d, mlp_tiles(M, g.w.k_in, g.r), X, sv, dY, M, dX, dA_g, dB_g, dA_u, dB_u, dA_d, dB_d,
                 ws, ws_bytes,
                 stream, early_grads);
}

// 16-bit entry points: bf16 base weights, always the staged-feed pair tile
// (the weight is already what the GEMM streams; nothing is dequantised).
size_t qlora_linear16_workspace_bytes(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (M <= 0 || K <= 0 || N <= 0 || !rank_ok(r, 4)) return 256;
  return linear_ws(M, K, N, r, false);
}
size_t qlora_mlp16_workspace_bytes(int64_t M, int64_t d, int64_t h, int32_t r) {
  if (M <= 0 || d <= 0 || h <= 0 || !rank_ok(r, 4)) return 256;
  return mlp_ws(M, d, h, r, false);
}
qlora_status qlora_linear16_fwd(const qlora_lora_linear16* lin, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                                qlora_bf16* XA_saved, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!lin) return QLORA_ERR_INVALID_ARG;
  const Lin l = lin_of(*lin);
  if (!l.w.w16) return QLORA_ERR_INVALID_ARG;
  return linear_fwd(&l, 4, X, M, Y, XA_saved, ws, ws_bytes, stream);
}
qlora_status qlora_linear16_bwd(const qlora_lora_linear16* lin, const qlora_bf16* X, const qlora_bf16* XA_saved,
                                const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB,
                                void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!lin) return QLORA_ERR_INVALID_ARG;
  const Lin l = lin_of(*lin);
  if (!l.w.w16) return QLORA_ERR_INVALID_ARG;
  return linear_bwd(&l, 4, X, XA_saved, dY, M, dX, dA, dB, ws, ws_bytes, stream);
}
qlora_status qlora_mlp16_fwd(qlora_act act, const qlora_lora_linear16* gate, const qlora_lora_linear16* up,
                             const qlora_lora_linear16* down, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                             const qlora_mlp_saved* sv, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!gate || !up || !down || !gate->w || !up->w || !down->w) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_fwd(act, &g, &u, &d, 4, X, M, Y, sv, ws, ws_bytes, stream);
}
qlora_status qlora_mlp16_bwd(qlora_act act, const qlora_lora_linear16* gate, const qlora_lora_linear16* up,
                             const qlora_lora_linear16* down, const qlora_bf16* X, const qlora_mlp_saved* sv,
                             const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                             qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d, void* ws,
                             size_t ws_bytes, qlora_stream_t stream) {
  if (!gate || !up || !down || !gate->w || !up->w || !down->w) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_bwd(act, &g, &u, &d, 4, X, sv, dY, M, dX, dA_g, dB_g, dA_u, dB_u, dA_d, dB_d, ws, ws_bytes, stream);
}
qlora_status qlora_mlp16_bwd_ev(qlora_act act, const qlora_lora_linear16* gate, const qlora_lora_linear16* up,
                                const qlora_lora_linear16* down, const qlora_bf16* X, const qlora_mlp_saved* sv,
                                const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                                qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d, void* ws,
                                size_t ws_bytes, qlora_stream_t stream, qlora_event_t early_grads) {
  if (!gate || !up || !down || !gate->w || !up->w || !down->w) return QLORA_ERR_INVALID_ARG;
  const Lin g = lin_of(*gate), u = lin_of(*up), d = lin_of(*down);
  return mlp_bwd(act, &g, &u, &d, 4, X, sv, dY, M, dX, dA_g, dB_g, dA_u, dB_u, dA_d, dB_d, ws, ws_bytes, stream,
                 early_grads);
}

qlora_status qlora_test_inject_timeout(void) {
  return cuda_status(arm_inject_timeout());
}

qlora_status qlora_last_device_status(void* ws, qlora_stream_t stream) {
  if (!ws) return QLORA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyAsync(ws, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  }
  if (v & QL_DEV_TIMEOUT) return QLORA_ERR_TIMEOUT;
  return v ? QLORA_ERR_DEVICE : QLORA_OK;
}

qlora_status qlora_trace_begin(void) {
  g_recs.clear();
  g_pool_used = 0;
  g_trace_only = -1;
  g_trace = true;
  return QLORA_OK;
}

qlora_status qlora_trace_begin_only(const char* kernel_name) {
  if (!kernel_name) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < K_COUNT; ++i) {
    if (std::strcmp(kernel_name, kKernelNames[i]) == 0) {
      qlora_status s = qlora_trace_begin();
      g_trace_only = i;
      return s;
    }
  }
  return QLORA_ERR_INVALID_ARG;
}

int32_t qlora_trace_end(qlora_trace_entry* out, int32_t max_entries) {
  g_trace = false;
  double tot[K_COUNT] = {0};
  int64_t cnt[K_COUNT] = {0};
  for (const TraceRec& r : g_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    tot[r.id] += ms;
    cnt[r.id] += 1;
  }
  g_recs.clear();
  int32_t n = 0;
  for (int i = 0; i < K_COUNT; ++i) {
    if (!cnt[i]) continue;
    if (out && n < max_entries) out[n] = {kKernelNames[i], cnt[i], tot[i]};
    ++n;
  }
  return n;
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward projection without a caller-supplied workspace.
//
// Some callers cannot hand us device memory: a kernel plugin that only receives
// the device pointers of its tensors from a host framework which owns all
// device memory (a raw cudaMalloc there would bypass the framework's allocator
// and memory budget), or a code path where allocating is not allowed at all.
// For them the scratch of qlora_linear_fwd (the status word, the s-scaled copy
// of X A and the split-K partial sums) lives in this fixed array instead.  Every
// GPU that loads the library holds it until the process exits.
static constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
static void* g_noalloc_scratch_ptr[64] = {};

// Device address of g_noalloc_scratch for the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
static qlora_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_CUDA;
  if (!g_noalloc_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
    g_noalloc_scratch_ptr[dev] = p;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return QLORA_OK;
}

extern "C" {

qlora_status qlora_linear_fwd_noalloc(const qlora_lora_linear* lin_nf4, const qlora_bf16* X, int64_t M,
                                      qlora_bf16* Y, qlora_bf16* XA_saved, qlora_stream_t stream) {
  if (!lin_nf4) return QLORA_ERR_INVALID_ARG;
  const Lin lv = lin_of(*lin_nf4);
  const Lin* lin = &lv;
  // The fixed scratch has no room for a staged weight: the staged configuration
  // falls back to the pair tile that dequantises in the mainloop (rank 16).
  const int tiles = (g_tiles == 0 || is_staged(g_tiles)) ? 2 : g_tiles;
  qlora_status s = check_linear(lin, tiles);
  if (s != QLORA_OK) return s;
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;
  if (!X || !Y || !XA_saved) return QLORA_ERR_INVALID_ARG;
  if (misaligned(X) || misaligned(Y) || misaligned(XA_saved)) return QLORA_ERR_MISALIGNED;
  if (M > kMaxDim) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t K = lin->w.k_in;
  const size_t vec = align256(static_cast<size_t>(M) * 32);
  // The X A pass normally splits its work over all resident CTAs, which can
  // give a 64-row group several partial sums.  When those do not fit, each
  // group goes to one CTA (one partial per group), so the scratch needed is
  // 256 + 32 M + 4096 ceil(M / 64) bytes (rounded up to 256) for any k_in.
  int target = 0;
  if (256 + vec + align256(rowproj_part_bytes(M, K, 16)) > kNoAllocScratchBytes)
    target = static_cast<int>(std::min<int64_t>(cdiv(M, 64), skinny_target_ctas(16)));
  const size_t need = 256 + vec + align256(rowproj_part_bytes(M, K, 16, target));
  if (need > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  void* base = nullptr;
  if ((s = noalloc_scratch(&base)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left; only the status word must start at zero.
  if (cudaMemsetAsync(base, 0, 256, st) != cudaSuccess) return QLORA_ERR_CUDA;
  char* w = static_cast<char*>(base);
  int* status = reinterpret_cast<int*>(w);
  bf16* xa = reinterpret_cast<bf16*>(XA_saved);
  bf16* XAs = lin->scale != 1.0f ? reinterpret_cast<bf16*>(w + 256) : xa;
  float* part = reinterpret_cast<float*>(w + 256 + vec);
  s = pass_rowproj(reinterpret_cast<const bf16*>(X), M, K, reinterpret_cast<const bf16*>(lin->A), nullptr, 16, part,
                   routs(rout(xa, 0, 16, 16, 0, 1.f), rout(XAs != xa ? XAs : nullptr, 0, 16, 16, 0, lin->scale)),
                   status, st, nullptr, target);
  if (s != QLORA_OK) return s;
  return gemm_fwd(*lin, reinterpret_cast<const bf16*>(X), M, XAs, reinterpret_cast<bf16*>(Y), status, tiles, nullptr,
                  st);
}

}  // extern "C"
