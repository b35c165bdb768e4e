// NF4 block quantisation (one-time) and the standalone, HBM-bound dequantiser.
//
// Format (QLoRA NormalFloat, linked from the Show HN thread "80% faster, 50%
// less memory, 0% loss of accuracy Llama finetuning"; the Mistral blog's
// benchmark quantises every projection with it): blocks of 64 consecutive
// elements along k_in of the row-major [n_out, k_in] weight, one binary32
// absmax per block, two 4-bit level indices per byte with the even element in
// the high nibble.  Dequantisation goes straight to bf16 (Mistral blog, item
// "2. Bitsandbytes bfloat16"): w = RNE_bf16(level[q] * absmax).
#include "kernels.cuh"
#include "ptx.cuh"

namespace ql {

// NF4 levels (binary32 bit patterns), ascending; level 7 is exactly 0.
__constant__ uint32_t c_nf4_bits[16] = {0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
                                        0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
                                        0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};
extern const uint32_t h_nf4_bits[16];
const uint32_t h_nf4_bits[16] = {0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
                                 0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
                                 0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};

// Level index of v = w / absmax (binary32): the number of level midpoints
// strictly below v.  The midpoints m_i = (c_i + c_{i+1}) / 2 are exact in
// binary64; with t_i = m_i rounded toward -inf to binary32, a binary32 v has
// v > m_i exactly when v > t_i (if m_i is a binary32 value, t_i = m_i; if
// not, t_i < m_i < the next binary32 after t_i, and v cannot lie strictly
// between those two).  So the comparisons run in binary32 against t and take
// the same decisions as the binary64 ones, ties (v = m_i) to the lower level
// included.  Four comparisons: a binary search over the 15 thresholds.
QL_DEV int nf4_level_index(float v, const float* t) {
  int q = v > t[7] ? 8 : 0;
  q += v > t[q + 3] ? 4 : 0;
  q += v > t[q + 1] ? 2 : 0;
  q += v > t[q] ? 1 : 0;
  return q;
}

// Eight threads per 64-element block (one 16-byte load of 8 bf16 each), eight
// blocks per warp.  absmax = max |w| (exact: bf16 values are binary32 values);
// v = w / absmax rounded once to binary32 (IEEE division); absmax 0 -> level 7.
// Each thread stores its 8 level indices as 4 bytes (even element in the high
// nibble) and the block's first thread its absmax.
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const bf16* __restrict__ w, int64_t nblocks,
                                                           uint8_t* __restrict__ codes, float* __restrict__ absmax) {
  __shared__ float thr[15];
  if (threadIdx.x < 15) {
    const double mid = 0.5 * (static_cast<double>(__uint_as_float(c_nf4_bits[threadIdx.x])) +
                              static_cast<double>(__uint_as_float(c_nf4_bits[threadIdx.x + 1])));
    thr[threadIdx.x] = __double2float_rd(mid);
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t blk = t >> 3;
  const int part = static_cast<int>(t & 7);
  const bool valid = blk < nblocks;
  uint4 raw = make_uint4(0, 0, 0, 0);
  if (valid) raw = __ldg(reinterpret_cast<const uint4*>(w + blk * 64 + part * 8));
  const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
  float x[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16_lo(wv[i]);
    x[2 * i + 1] = bf16_hi(wv[i]);
  }
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
  // the block's eight threads are lanes 8j .. 8j + 7 of one warp
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (!valid) return;
  uint32_t packed = 0x77777777u;  // all-zero block: level 7 everywhere
  if (m > 0.f) {
    packed = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = nf4_level_index(__fdiv_rn(x[i], m), thr);
      // element 2b in the high nibble of byte b, element 2b + 1 in its low nibble
      packed |= static_cast<uint32_t>(q) << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
    }
  }
  reinterpret_cast<uint32_t*>(codes + blk * 32)[part] = packed;
  if (part == 0) absmax[blk] = m;
}

// Dequantisation of up to three tensors in one launch.  A warp takes runs of
// 1024 elements: lane l expands the 8 elements at 8l + 256i (i = 0..3), so
// each warp-wide load of codes is 128 contiguous bytes and each bf16 store
// 512 contiguous bytes.  The 16 levels sit in shared memory (lanes reading
// the same level are served by one broadcast).
struct DqJob {
  const uint8_t* codes;
  const float* absmax;
  bf16* out;
  int64_t runs;  // numel / 1024, rounded up
  int64_t numel;
};
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(const DqJob j0, const DqJob j1, const DqJob j2) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = __uint_as_float(c_nf4_bits[threadIdx.x]);
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t r01 = j0.runs + j1.runs, total = r01 + j2.runs;
  for (int64_t run = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; run < total; run += warps) {
    const int which = run < j0.runs ? 0 : (run < r01 ? 1 : 2);
    const int64_t base = (run - (which == 0 ? 0 : (which == 1 ? j0.runs : r01))) * 1024;
    const uint8_t* codes = which == 0 ? j0.codes : (which == 1 ? j1.codes : j2.codes);
    const float* absmax = which == 0 ? j0.absmax : (which == 1 ? j1.absmax : j2.absmax);
    bf16* out = which == 0 ? j0.out : (which == 1 ? j1.out : j2.out);
    const int64_t numel = which == 0 ? j0.numel : (which == 1 ? j1.numel : j2.numel);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t e = base + i * 256 + lane * 8;
      if (e >= numel) break;
      const uint32_t c = __ldg(reinterpret_cast<const uint32_t*>(codes + (e >> 1)));
      const float a = __ldg(absmax + (e >> 6));
      uint32_t o[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (c >> (8 * b)) & 0xFFu;
        o[b] = pack_bf16x2(lut[byte >> 4] * a, lut[byte & 0xF] * a);
      }
      *reinterpret_cast<uint4*>(out + e) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

cudaError_t launch_nf4_quantize(const bf16* w, int64_t numel, uint8_t* codes, float* absmax, cudaStream_t st) {
  const int64_t nblocks = numel / 64;
  const int64_t threads = nblocks * 8;
  const int64_t grid = (threads + 255) / 256;
  return launch_pdl(nf4_quantize_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, w, nblocks, codes,
                    absmax);
}

// Dequantises n = 1 to 3 tensors in one launch: tensor i has numel[i] elements,
// its codes and absmax, and goes to out[i].
cudaError_t launch_nf4_dequantize(const uint8_t* const* codes, const float* const* absmax, const int64_t* numel,
                                  bf16* const* out, int n, cudaStream_t st, int num_sms) {
  if (n < 1 || n > 3) return cudaErrorInvalidValue;
  DqJob j[3] = {};
  for (int i = 0; i < n; ++i) j[i] = {codes[i], absmax[i], out[i], (numel[i] + 1023) / 1024, numel[i]};
  int64_t grid = (j[0].runs + j[1].runs + j[2].runs + 7) / 8;  // one run per warp, 8 warps per CTA
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;  // 8 CTAs of 256 threads per SM
  if (grid > cap) grid = cap;
  grid = apply_grid_cap(static_cast<int>(grid), 1);
  if (grid < 1) grid = 1;
  return launch_pdl(nf4_dequantize_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, j[0], j[1], j[2]);
}

}  // namespace ql
