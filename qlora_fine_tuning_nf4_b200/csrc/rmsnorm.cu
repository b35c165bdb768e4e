// RMS layer norm, forward and backward (Mistral blog, table "逐项性能拆解"
// item "8. 快速 RMS Layernorm"; Gemma blog "+1 to RMS LayerNorm"):
//   rstd = 1 / sqrt(mean_j x_j^2 + eps),  y = x * rstd * g,  g = w or 1 + w,
//   dx_j = rstd * (g_j dy_j - n_j * mean_i(n_i g_i dy_i)),  n = x * rstd,
// with the norm weight frozen.  HBM-bound row kernels.  Rows up to 8192 wide:
// one 128-thread CTA per row holds the row in registers (16-byte loads, all in
// flight at once, one pass over DRAM) and reduces its fp32 statistics in a
// fixed order (deterministic).  Wider rows: one warp per row, two passes, the
// second served from the cache.
#include "kernels.cuh"
#include "ptx.cuh"

namespace ql {

constexpr int NORM_WARPS = 8;

QL_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
QL_DEV void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_lo(w[i]);
    f[2 * i + 1] = bf16_hi(w[i]);
  }
}
QL_DEV void gain8(const bf16* w, int c, int plus_one, float (&g)[8]) {
  unpack8(__ldg(reinterpret_cast<const uint4*>(w + c)), g);
  if (plus_one) {
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] += 1.0f;
  }
}

__global__ void __launch_bounds__(32 * NORM_WARPS) rmsnorm_fwd_kernel(const bf16* __restrict__ X,
                                                                      const bf16* __restrict__ w, int M, int d,
                                                                      float eps, int plus_one, bf16* __restrict__ Y,
                                                                      float* __restrict__ rstd_out) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * NORM_WARPS + (threadIdx.x >> 5);
  if (row >= M) return;
  const bf16* x = X + static_cast<size_t>(row) * d;
  float ss = 0.f;
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(x + c)), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  ss = warp_sum(ss);
  const float rstd = __fdiv_rn(1.0f, sqrtf(__fdiv_rn(ss, static_cast<float>(d)) + eps));
  bf16* y = Y + static_cast<size_t>(row) * d;
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8], g[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(x + c)), f);
    gain8(w, c, plus_one, g);
    uint4 o;
    o.x = pack_bf16x2(f[0] * rstd * g[0], f[1] * rstd * g[1]);
    o.y = pack_bf16x2(f[2] * rstd * g[2], f[3] * rstd * g[3]);
    o.z = pack_bf16x2(f[4] * rstd * g[4], f[5] * rstd * g[5]);
    o.w = pack_bf16x2(f[6] * rstd * g[6], f[7] * rstd * g[7]);
    *reinterpret_cast<uint4*>(y + c) = o;
  }
  if (lane == 0) rstd_out[row] = rstd;
}

__global__ void __launch_bounds__(32 * NORM_WARPS) rmsnorm_bwd_kernel(const bf16* __restrict__ X,
                                                                      const bf16* __restrict__ w,
                                                                      const float* __restrict__ rstd_in,
                                                                      const bf16* __restrict__ dY, int M, int d,
                                                                      int plus_one, bf16* __restrict__ dX) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * NORM_WARPS + (threadIdx.x >> 5);
  if (row >= M) return;
  const size_t off = static_cast<size_t>(row) * d;
  const float rstd = rstd_in[row];
  float acc = 0.f;  // sum_i x_i g_i dy_i
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8], g[8], dy[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(X + off + c)), f);
    unpack8(__ldg(reinterpret_cast<const uint4*>(dY + off + c)), dy);
    gain8(w, c, plus_one, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = fmaf(f[i] * g[i], dy[i], acc);
  }
  acc = warp_sum(acc);
  // mean_i(n_i g_i dy_i) = rstd * acc / d;  dx_j = rstd * (g_j dy_j - x_j * rstd * that)
  const float cm = rstd * rstd * __fdiv_rn(acc, static_cast<float>(d));
#pragma unroll 4
  for (int c = lane * 8; c < d; c += 256) {
    float f[8], g[8], dy[8], o[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(X + off + c)), f);
    unpack8(__ldg(reinterpret_cast<const uint4*>(dY + off + c)), dy);
    gain8(w, c, plus_one, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = rstd * (g[i] * dy[i] - f[i] * cm);
    uint4 u;
    u.x = pack_bf16x2(o[0], o[1]);
    u.y = pack_bf16x2(o[2], o[3]);
    u.z = pack_bf16x2(o[4], o[5]);
    u.w = pack_bf16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(dX + off + c) = u;
  }
}

// ------------------------------------------------- row-in-registers path --
constexpr int NR_THREADS = 128;
constexpr int NR_MAXCH = 8;  // 16-byte chunks per thread: rows up to 128 * 8 * 8 = 8192 wide

// Sum over the CTA's 128 threads: warp butterflies, then the four warp sums in order.
QL_DEV float cta_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5;
  __syncthreads();  // red[] is free (a previous reduction has been read)
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

__global__ void __launch_bounds__(NR_THREADS) rmsnorm_fwd_row_kernel(const bf16* __restrict__ X,
                                                                     const bf16* __restrict__ w, int d, float eps,
                                                                     int plus_one, bf16* __restrict__ Y,
                                                                     float* __restrict__ rstd_out) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float red[4];
  const int row = blockIdx.x;
  const bf16* x = X + static_cast<size_t>(row) * d;
  uint4 v[NR_MAXCH];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    const int c = (i * NR_THREADS + threadIdx.x) * 8;
    v[i] = c < d ? __ldg(reinterpret_cast<const uint4*>(x + c)) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    float f[8];
    unpack8(v[i], f);
#pragma unroll
    for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
  }
  ss = cta_sum(ss, red);
  const float rstd = __fdiv_rn(1.0f, sqrtf(__fdiv_rn(ss, static_cast<float>(d)) + eps));
  bf16* y = Y + static_cast<size_t>(row) * d;
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    const int c = (i * NR_THREADS + threadIdx.x) * 8;
    if (c >= d) break;
    float f[8], g[8];
    unpack8(v[i], f);
    gain8(w, c, plus_one, g);
    uint4 o;
    o.x = pack_bf16x2(f[0] * rstd * g[0], f[1] * rstd * g[1]);
    o.y = pack_bf16x2(f[2] * rstd * g[2], f[3] * rstd * g[3]);
    o.z = pack_bf16x2(f[4] * rstd * g[4], f[5] * rstd * g[5]);
    o.w = pack_bf16x2(f[6] * rstd * g[6], f[7] * rstd * g[7]);
    *reinterpret_cast<uint4*>(y + c) = o;
  }
  if (threadIdx.x == 0) rstd_out[row] = rstd;
}

__global__ void __launch_bounds__(NR_THREADS) rmsnorm_bwd_row_kernel(const bf16* __restrict__ X,
                                                                     const bf16* __restrict__ w,
                                                                     const float* __restrict__ rstd_in,
                                                                     const bf16* __restrict__ dY, int d, int plus_one,
                                                                     bf16* __restrict__ dX) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float red[4];
  const int row = blockIdx.x;
  const size_t off = static_cast<size_t>(row) * d;
  const float rstd = rstd_in[row];
  uint4 xv[NR_MAXCH], dv[NR_MAXCH];
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    const int c = (i * NR_THREADS + threadIdx.x) * 8;
    const bool in = c < d;
    xv[i] = in ? __ldg(reinterpret_cast<const uint4*>(X + off + c)) : make_uint4(0, 0, 0, 0);
    dv[i] = in ? __ldg(reinterpret_cast<const uint4*>(dY + off + c)) : make_uint4(0, 0, 0, 0);
  }
  float acc = 0.f;  // sum_i x_i g_i dy_i
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    const int c = (i * NR_THREADS + threadIdx.x) * 8;
    if (c >= d) break;
    float f[8], g[8], dy[8];
    unpack8(xv[i], f);
    unpack8(dv[i], dy);
    gain8(w, c, plus_one, g);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = fmaf(f[k] * g[k], dy[k], acc);
  }
  acc = cta_sum(acc, red);
  const float cm = rstd * rstd * __fdiv_rn(acc, static_cast<float>(d));
#pragma unroll
  for (int i = 0; i < NR_MAXCH; ++i) {
    const int c = (i * NR_THREADS + threadIdx.x) * 8;
    if (c >= d) break;
    float f[8], g[8], dy[8], o[8];
    unpack8(xv[i], f);
    unpack8(dv[i], dy);
    gain8(w, c, plus_one, g);
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = rstd * (g[k] * dy[k] - f[k] * cm);
    uint4 u;
    u.x = pack_bf16x2(o[0], o[1]);
    u.y = pack_bf16x2(o[2], o[3]);
    u.z = pack_bf16x2(o[4], o[5]);
    u.w = pack_bf16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(dX + off + c) = u;
  }
}

cudaError_t launch_rmsnorm_fwd(const bf16* X, const bf16* w, int M, int d, float eps, int plus_one, bf16* Y,
                               float* rstd, cudaStream_t st) {
  if (d <= NR_THREADS * NR_MAXCH * 8) {
    return launch_pdl(rmsnorm_fwd_row_kernel, dim3(M), dim3(NR_THREADS), 0, st, X, w, d, eps, plus_one, Y, rstd);
  }
  return launch_pdl(rmsnorm_fwd_kernel, dim3((M + NORM_WARPS - 1) / NORM_WARPS), dim3(32 * NORM_WARPS), 0, st, X, w,
                    M, d, eps, plus_one, Y, rstd);
}

cudaError_t launch_rmsnorm_bwd(const bf16* X, const bf16* w, const float* rstd, const bf16* dY, int M, int d,
                               int plus_one, bf16* dX, cudaStream_t st) {
  if (d <= NR_THREADS * NR_MAXCH * 8) {
    return launch_pdl(rmsnorm_bwd_row_kernel, dim3(M), dim3(NR_THREADS), 0, st, X, w, rstd, dY, d, plus_one, dX);
  }
  return launch_pdl(rmsnorm_bwd_kernel, dim3((M + NORM_WARPS - 1) / NORM_WARPS), dim3(32 * NORM_WARPS), 0, st, X, w,
                    rstd, dY, M, d, plus_one, dX);
}

}  // namespace ql
