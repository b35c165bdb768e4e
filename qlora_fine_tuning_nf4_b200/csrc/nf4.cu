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

// One warp per 64-element block: lane l owns elements 2l and 2l+1.
// absmax = max |w| (exact); v = w / absmax rounded once to binary32; the
// level index is the number of midpoints (exact in binary64) strictly below
// v, so a value on a midpoint takes the lower level; absmax 0 -> level 7.
__global__ void nf4_quantize_kernel(const bf16* __restrict__ w, int64_t nblocks, uint8_t* __restrict__ codes,
                                    float* __restrict__ absmax) {
  const int64_t blk = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (blk >= nblocks) return;
  const uint32_t pair = reinterpret_cast<const uint32_t*>(w + blk * 64)[lane];
  const float x0 = __uint_as_float(pair << 16), x1 = __uint_as_float(pair & 0xFFFF0000u);
  float m = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int q0 = 7, q1 = 7;
  if (m > 0.f) {
    const double v0 = static_cast<double>(__fdiv_rn(x0, m));
    const double v1 = static_cast<double>(__fdiv_rn(x1, m));
    q0 = 0;
    q1 = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) {
      const double mid = 0.5 * (static_cast<double>(__uint_as_float(c_nf4_bits[i])) +
                                static_cast<double>(__uint_as_float(c_nf4_bits[i + 1])));
      q0 += v0 > mid;
      q1 += v1 > mid;
    }
  }
  codes[blk * 32 + lane] = static_cast<uint8_t>((q0 << 4) | q1);
  if (lane == 0) absmax[blk] = m;
}

// Each warp handles runs of 1024 elements: lane l takes 8 consecutive
// elements at offsets 8l + 256i (i = 0..3), so every warp-wide load of codes
// is 128 contiguous bytes and every store of bf16 is 512 contiguous bytes.
__global__ void nf4_dequantize_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ absmax,
                                      int64_t numel, bf16* __restrict__ out) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = __uint_as_float(c_nf4_bits[threadIdx.x]);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  for (int64_t base = wid * 1024; base < numel; base += warps * 1024) {
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
  const int64_t threads = nblocks * 32;
  const int64_t grid = (threads + 255) / 256;
  nf4_quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(w, nblocks, codes, absmax);
  return cudaGetLastError();
}

cudaError_t launch_nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t numel, bf16* out,
                                  cudaStream_t st, int num_sms) {
  const int64_t chunks = (numel + 1023) / 1024;  // one warp-run each
  int64_t grid = (chunks + 7) / 8;               // 8 warps per CTA
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_dequantize_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(codes, absmax, numel, out);
  return cudaGetLastError();
}

}  // namespace ql
