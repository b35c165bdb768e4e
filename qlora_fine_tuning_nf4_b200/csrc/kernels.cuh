// Kernel-side argument structs and launch helpers shared by the .cu files of
// libqlora.  Host code fills these; kernels only read them.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ql {

using bf16 = __nv_bfloat16;

// Upper bound on the CTAs of every persistent launch (GEMM, skinny passes,
// weight dequantisation); 0 = none.  Set only by the test hook
// qlora_test_set_grid_cap, so that small problems make every CTA (pair) walk
// several tiles or work units.
extern int g_grid_cap;
inline int apply_grid_cap(int ctas, int multiple) {
  if (g_grid_cap <= 0 || ctas <= g_grid_cap) return ctas;
  const int c = g_grid_cap - g_grid_cap % multiple;
  return c > multiple ? c : multiple;
}

// ------------------------------------------------------------------ GEMM ---
// D = A * op(dequant(W)) + LoRA, on tcgen05 tensor cores.
//   MODE_FWD:     reduction over k_in, W [N, K] is the K-major B operand.
//   MODE_FWD_GLU: as MODE_FWD with two weights (gate | up) side by side in
//                 one 256-wide N tile; epilogue forms the gated activation.
//   MODE_BWD:     reduction over n_out, W [N, K] is the MN-major B operand
//                 (dX = dY W); up to two reduction segments (concatenated K).
enum GemmMode : int { MODE_FWD = 0, MODE_FWD_GLU = 1, MODE_BWD = 2 };
enum GemmEpi : int { EPI_STORE = 0, EPI_GLU_FWD = 1, EPI_GLU_BWD = 2 };
enum Act : int { ACT_SILU = 0, ACT_GELU_TANH = 1 };

struct GemmMaps {
  CUtensorMap a[2];       // A operand per segment: bf16 [M, Kseg], box {64,128}, 128B swizzle
  CUtensorMap codes[2];   // NF4 codes (per segment, or gate/up half for MODE_FWD_GLU)
  CUtensorMap absmax[2];  // fp32 absmax, matching codes[]
  CUtensorMap la[3];      // LoRA left operand(s): s*XA or s*G [M, r]
  CUtensorMap lb[3];      // LoRA right operand(s): B [r, N] (forward) or A [N, r] (backward)
  CUtensorMap b[2];       // staged feed only: the dequantised bf16 weight, matching codes[]
  CUtensorMap out[3];     // staged feed only: outputs (D | E, G, H | dE, dG), box {32,32}, 64B swizzle
};

struct GemmArgs {
  int M;        // rows of A and of the output
  int N;        // output columns (MODE_FWD_GLU: h, the width of E/G/H)
  int nkb0;     // 64-wide reduction blocks in segment 0
  int nkb1;     // ... in segment 1 (0 if one segment)
  int lora;     // number of LoRA operands (0..3; MODE_FWD: 1, chosen per tile by ncut)
  int lora_k16; // staged feed: 16-wide reduction steps per LoRA operand (rank / 16, 1..4)
  int ncut[2];  // MODE_FWD, staged feed: output columns [0, ncut0) take LoRA operand 0,
                // [ncut0, ncut1) operand 1, the rest operand 2 (fused projections); 0 = no cut
  int act;      // Act
  int ldo;      // leading dimension (elements) of all outputs / epilogue inputs
  bf16* D;      // EPI_STORE output [M, N]
  bf16* E;      // EPI_GLU_FWD outputs [M, N]: e, g and h = act(e) * g
  bf16* G;
  bf16* H;
  const bf16* Ein;  // EPI_GLU_BWD inputs: saved e and g
  const bf16* Gin;
  bf16* dE;     // EPI_GLU_BWD outputs
  bf16* dG;
  int* status;  // device status word (timeouts)
  int group_m;  // tile order: groups of group_m output-row tiles, rows fastest inside a group (>= 1)
};

// --------------------------------------------------------------- skinny ---
// Rank-r products on warp-level mma.sync.  Each skinny kernel is persistent:
// its P CTAs split the work units (64 x 64 tiles, or 64-row x 256-column
// blocks) into P contiguous, equally sized ranges, so every CTA streams the
// same number of bytes.  A CTA writes one fp32 partial per output group
// (a 64-row or 256-column block of the result) it touches; a reduction kernel
// adds each group's partials in slot order (deterministic).

// Balanced contiguous partition of U units over P parts: part c owns
// [part_begin(c), part_begin(c + 1)); part_owner(u) is the part that owns u.
__host__ __device__ inline int part_begin(int c, int U, int P) {
  return static_cast<int>(static_cast<int64_t>(c) * U / P);
}
__host__ __device__ inline int part_owner(int u, int U, int P) {
  return static_cast<int>(((static_cast<int64_t>(u) + 1) * P - 1) / U);
}

// Partition of a skinny pass: U super-units of `align` units each over P CTAs;
// output group g covers units [g * upg, (g + 1) * upg).
struct SkPart {
  int U, P, align, upg;
};
// CTA owning unit u, first slot CTA of group g, and number of slots of group g
__host__ __device__ inline int sk_owner(const SkPart& p, int u) { return part_owner(u / p.align, p.U, p.P); }
__host__ __device__ inline int sk_first(const SkPart& p, int g) { return sk_owner(p, g * p.upg); }
__host__ __device__ inline int sk_slots(const SkPart& p, int g) {
  return sk_owner(p, g * p.upg + p.upg - 1) - sk_first(p, g) + 1;
}

// Output of the partial-sum reduction: `width` of the R partial columns,
// scaled, rounded to bf16 and written row-major or transposed.
struct ReduceOut {
  bf16* ptr;      // destination (nullptr = unused)
  int col0;       // first of the partial columns this output takes
  int width;      // number of partial columns it takes (the LoRA rank)
  int ld;         // row stride of the destination (elements)
  int transpose;  // 0: dst[row * ld + c], 1: dst[c * ld + row]
  float scale;
};
struct ReduceOuts {
  ReduceOut o[4];
};

// Partials of one output of a skinny pass: part[g][slot][row in group][R] for
// `groups` groups of `grows` rows (the last may extend past `rows`), slot_cap
// slots per group; group g has `nslots` slots if nslots > 0, else
// sk_slots(sp, g).  The reduction adds them in slot order and stores `outs`.
struct ReduceJob {
  float* part;
  int groups, grows, rows, R, slot_cap, nslots;
  SkPart sp;
  ReduceOuts outs;
  int* status;  // device status word (the checked build's bounds checks report there)
};

// Reductions one launch of the reduction kernel can serve.
constexpr int kMaxReduceJobs = 6;

// Launch with programmatic stream serialisation (the kernel calls
// grid_dep_wait() before reading what earlier kernels wrote).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace ql
