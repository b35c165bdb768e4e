// Rank-r ("skinny") products of the LoRA path on warp-level mma.sync.
//
// The Mistral blog ("用 Unsloth 微调 Mistral，速度提升 14 倍", item
// "10、11. 手动 Autograd") brackets every chained product so that the rank-r
// factor is contracted first; these kernels are those contractions:
//   rowproj   P[m, :]  = T[m, :] V          V = [K, 16*NV] (LoRA A)     X A, H A_d
//   colproj   Q[n, :]  = T[:, n]^T U        U = [M, R]                   X^T G (dA)
//   dypass    G[m, :]  = T[m, :] B^T  and  Q[n, :] = T[:, n]^T U          dY B^T, (X A)^T dY
// Each CTA streams 64x64 bf16 tiles of T through a TMA/mbarrier ring (the
// kernels are HBM-bound on T) and writes fp32 partial sums over its slice of
// the reduction; `reduce_partials_kernel` adds the slices in a fixed order,
// applies the LoRA scale and rounds to bf16, so results are deterministic.
#include "kernels.cuh"
#include "ptx.cuh"

namespace ql {

constexpr int SK_THREADS = 128;
constexpr int SK_STAGES = 4;
constexpr int T_TILE = 64 * 64 * 2;  // bytes

// A-fragment (16x16) of rows [r0, r0+16) and cols [c0, c0+16) of a 64x64
// 128B-swizzled tile (row-major, 128 bytes per row).
QL_DEV void frag_a_rows(uint32_t tile, int r0, int c0, int lane, uint32_t (&a)[4]) {
  const int row = r0 + (lane & 15);
  const int chunk = (c0 >> 3) + (lane >> 4);
  ldsm_x4(tile + row * 128 + ((chunk ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
}
// A-fragment of the TRANSPOSED tile: rows = tile columns [n0, n0+16),
// reduction = tile rows [m0, m0+16).
QL_DEV void frag_a_cols(uint32_t tile, int m0, int n0, int lane, uint32_t (&a)[4]) {
  const int j = lane >> 3, i = lane & 7;
  const int m = m0 + ((j >> 1) << 3) + i;
  const int chunk = (n0 >> 3) + (j & 1);
  ldsm_x4_t(tile + m * 128 + ((chunk ^ (m & 7)) << 4), a[0], a[1], a[2], a[3]);
}
// B-fragment (16x8) from a row-major [k][n] tile with `row_bytes` per row
// (no swizzle): reduction rows [k0, k0+16), columns [n0, n0+8).
QL_DEV void frag_b_kn(uint32_t tile, int row_bytes, int k0, int n0, int lane, uint32_t (&b)[2]) {
  const int k = k0 + (lane & 15);
  ldsm_x2_t(tile + k * row_bytes + n0 * 2, b[0], b[1]);
}
// B-fragment from a 128B-swizzled [n][k] tile (rows = output column n,
// 128 bytes of k per row): reduction [k0, k0+16), columns [n0, n0+8).
QL_DEV void frag_b_nk(uint32_t tile, int k0, int n0, int lane, uint32_t (&b)[2]) {
  const int n = n0 + (lane & 7);
  const int chunk = (k0 >> 3) + ((lane >> 3) & 1);
  ldsm_x2(tile + n * 128 + ((chunk ^ (n & 7)) << 4), b[0], b[1]);
}

// Uniform bounded wait for all threads of the CTA.
QL_DEV bool cta_wait(uint32_t bar, uint32_t parity, int* status) {
  const bool ok = mbar_wait(bar, parity, status);
  return __syncthreads_and(ok) != 0;
}

// ------------------------------------------------------------- rowproj ---
// part[ks][m][16*NV] = sum over this CTA's k-slice of T[m,k] * V_j[k, :]
template <int NV>
__global__ void __launch_bounds__(SK_THREADS) rowproj_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                             const __grid_constant__ CUtensorMap tmap_v0,
                                                             const __grid_constant__ CUtensorMap tmap_v1,
                                                             float* __restrict__ part, int M, int K, int kb_per_split,
                                                             int* status) {
  constexpr int R = 16 * NV;
  constexpr int V_TILE = 64 * 16 * 2;
  constexpr int STAGE = T_TILE + NV * V_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 64;
  const int ks = blockIdx.y;
  const int kb0 = ks * kb_per_split;
  const int nkb = min(K / 64 - kb0, kb_per_split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int it) {
    const int s = it % SK_STAGES;
    const uint32_t st = sbase + s * STAGE;
    mbar_arrive_expect_tx(bars + 8 * s, STAGE);
    const int k = (kb0 + it) * 64;
    tma_load_2d(st, &tmap_t, bars + 8 * s, k, m0);
    tma_load_2d(st + T_TILE, &tmap_v0, bars + 8 * s, 0, k);
    if (NV == 2) tma_load_2d(st + T_TILE + V_TILE, &tmap_v1, bars + 8 * s, 0, k);
  };
  if (threadIdx.x == 0)
    for (int it = 0; it < SK_STAGES && it < nkb; ++it) issue(it);

  float acc[R / 8][4] = {};
  for (int it = 0; it < nkb; ++it) {
    const int s = it % SK_STAGES;
    if (!cta_wait(bars + 8 * s, (it / SK_STAGES) & 1, status)) return;
    const uint32_t t = sbase + s * STAGE;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      frag_a_rows(t, warp * 16, kk * 16, lane, a);
#pragma unroll
      for (int nb = 0; nb < R / 8; ++nb) {
        uint32_t b[2];
        frag_b_kn(t + T_TILE + (nb >> 1) * V_TILE, 32, kk * 16, (nb & 1) * 8, lane, b);
        mma_bf16_16816(acc[nb], a[0], a[1], a[2], a[3], b[0], b[1]);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && it + SK_STAGES < nkb) issue(it + SK_STAGES);
  }
  const int r_lo = m0 + warp * 16 + (lane >> 2);
  float* base = part + static_cast<size_t>(ks) * M * R;
#pragma unroll
  for (int nb = 0; nb < R / 8; ++nb) {
    const int c = nb * 8 + (lane & 3) * 2;
    if (r_lo < M) *reinterpret_cast<float2*>(base + static_cast<size_t>(r_lo) * R + c) = make_float2(acc[nb][0], acc[nb][1]);
    if (r_lo + 8 < M)
      *reinterpret_cast<float2*>(base + static_cast<size_t>(r_lo + 8) * R + c) = make_float2(acc[nb][2], acc[nb][3]);
  }
}

// ------------------------------------------------------------- colproj ---
// part[ms][n][R] = sum over this CTA's m-slice of T[m,n] * U[m, :]
template <int R>
__global__ void __launch_bounds__(SK_THREADS) colproj_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                             const __grid_constant__ CUtensorMap tmap_u,
                                                             float* __restrict__ part, int M, int N, int mb_per_split,
                                                             int* status) {
  constexpr int U_TILE = 64 * R * 2;
  constexpr int STAGE = T_TILE + U_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 64;
  const int ms = blockIdx.y;
  const int mb0 = ms * mb_per_split;
  const int nmb = min((M + 63) / 64 - mb0, mb_per_split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int it) {
    const int s = it % SK_STAGES;
    const uint32_t st = sbase + s * STAGE;
    mbar_arrive_expect_tx(bars + 8 * s, STAGE);
    const int m = (mb0 + it) * 64;
    tma_load_2d(st, &tmap_t, bars + 8 * s, n0, m);
    tma_load_2d(st + T_TILE, &tmap_u, bars + 8 * s, 0, m);
  };
  if (threadIdx.x == 0)
    for (int it = 0; it < SK_STAGES && it < nmb; ++it) issue(it);

  float acc[R / 8][4] = {};
  for (int it = 0; it < nmb; ++it) {
    const int s = it % SK_STAGES;
    if (!cta_wait(bars + 8 * s, (it / SK_STAGES) & 1, status)) return;
    const uint32_t t = sbase + s * STAGE;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      frag_a_cols(t, kk * 16, warp * 16, lane, a);
#pragma unroll
      for (int nb = 0; nb < R / 8; ++nb) {
        uint32_t b[2];
        frag_b_kn(t + T_TILE, R * 2, kk * 16, nb * 8, lane, b);
        mma_bf16_16816(acc[nb], a[0], a[1], a[2], a[3], b[0], b[1]);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && it + SK_STAGES < nmb) issue(it + SK_STAGES);
  }
  const int n_lo = n0 + warp * 16 + (lane >> 2);
  float* base = part + static_cast<size_t>(ms) * N * R;
#pragma unroll
  for (int nb = 0; nb < R / 8; ++nb) {
    const int c = nb * 8 + (lane & 3) * 2;
    if (n_lo < N) *reinterpret_cast<float2*>(base + static_cast<size_t>(n_lo) * R + c) = make_float2(acc[nb][0], acc[nb][1]);
    if (n_lo + 8 < N)
      *reinterpret_cast<float2*>(base + static_cast<size_t>(n_lo + 8) * R + c) = make_float2(acc[nb][2], acc[nb][3]);
  }
}

// -------------------------------------------------------------- dypass ---
// One read of T = dY [M, N] gives both
//   gpart[ns][m][16] = sum over this CTA's columns of T[m,n] * Bl[:, n]   (Bl = LoRA B, [16, N])
//   qpart[ms][n][16] = sum over this CTA's rows    of T[m,n] * U[m, :]    (U = X A, [M, 16])
// CTA tile: RC x 64 rows by CC x 64 columns, visited row-chunk major.
template <int CC>
__global__ void __launch_bounds__(SK_THREADS) dypass_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                            const __grid_constant__ CUtensorMap tmap_u,
                                                            const __grid_constant__ CUtensorMap tmap_b,
                                                            float* __restrict__ gpart, float* __restrict__ qpart,
                                                            int M, int N, int rc_per_cta, int* status) {
  constexpr int U_TILE = 64 * 16 * 2;
  constexpr int B_TILE = 16 * 64 * 2;
  constexpr int STAGE = T_TILE + U_TILE + B_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ns = blockIdx.x, ms = blockIdx.y;
  const int n0 = ns * CC * 64;
  const int m0 = ms * rc_per_cta * 64;
  const int nrc = min((M - m0 + 63) / 64, rc_per_cta);
  const int ncc = min((N - n0 + 63) / 64, CC);
  const int total = nrc * ncc;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int it) {
    const int s = it % SK_STAGES;
    const uint32_t st = sbase + s * STAGE;
    const int rc = it / ncc, cc = it % ncc;
    mbar_arrive_expect_tx(bars + 8 * s, STAGE);
    tma_load_2d(st, &tmap_t, bars + 8 * s, n0 + cc * 64, m0 + rc * 64);
    tma_load_2d(st + T_TILE, &tmap_u, bars + 8 * s, 0, m0 + rc * 64);
    tma_load_2d(st + T_TILE + U_TILE, &tmap_b, bars + 8 * s, n0 + cc * 64, 0);
  };
  if (threadIdx.x == 0)
    for (int it = 0; it < SK_STAGES && it < total; ++it) issue(it);

  float gacc[2][4];
  float qacc[CC][2][4] = {};
  for (int it = 0; it < total; ++it) {
    const int rc = it / ncc, cc = it % ncc;
    if (cc == 0) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) gacc[i][j] = 0.f;
    }
    const int s = it % SK_STAGES;
    if (!cta_wait(bars + 8 * s, (it / SK_STAGES) & 1, status)) return;
    const uint32_t t = sbase + s * STAGE;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      // G += T[rows 16w.., cols kk*16..] * Bl^T
      frag_a_rows(t, warp * 16, kk * 16, lane, a);
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        uint32_t b[2];
        frag_b_nk(t + T_TILE + U_TILE, kk * 16, nb * 8, lane, b);
        mma_bf16_16816(gacc[nb], a[0], a[1], a[2], a[3], b[0], b[1]);
      }
      // Q += T[rows kk*16.., cols 16w..]^T * U
      frag_a_cols(t, kk * 16, warp * 16, lane, a);
#pragma unroll
      for (int c = 0; c < CC; ++c) {
        if (c != cc) continue;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          uint32_t b[2];
          frag_b_kn(t + T_TILE, 32, kk * 16, nb * 8, lane, b);
          mma_bf16_16816(qacc[c][nb], a[0], a[1], a[2], a[3], b[0], b[1]);
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && it + SK_STAGES < total) issue(it + SK_STAGES);
    if (cc == ncc - 1) {
      const int r_lo = m0 + rc * 64 + warp * 16 + (lane >> 2);
      float* base = gpart + static_cast<size_t>(ns) * M * 16;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int c = nb * 8 + (lane & 3) * 2;
        if (r_lo < M) *reinterpret_cast<float2*>(base + static_cast<size_t>(r_lo) * 16 + c) = make_float2(gacc[nb][0], gacc[nb][1]);
        if (r_lo + 8 < M)
          *reinterpret_cast<float2*>(base + static_cast<size_t>(r_lo + 8) * 16 + c) = make_float2(gacc[nb][2], gacc[nb][3]);
      }
    }
  }
  float* qbase = qpart + static_cast<size_t>(ms) * N * 16;
#pragma unroll
  for (int c = 0; c < CC; ++c) {
    if (c >= ncc) break;
    const int n_lo = n0 + c * 64 + warp * 16 + (lane >> 2);
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      const int col = nb * 8 + (lane & 3) * 2;
      if (n_lo < N) *reinterpret_cast<float2*>(qbase + static_cast<size_t>(n_lo) * 16 + col) = make_float2(qacc[c][nb][0], qacc[c][nb][1]);
      if (n_lo + 8 < N)
        *reinterpret_cast<float2*>(qbase + static_cast<size_t>(n_lo + 8) * 16 + col) = make_float2(qacc[c][nb][2], qacc[c][nb][3]);
    }
  }
}

// ------------------------------------------------------------- reduce ----
// out = bf16(scale * sum_{s < S} part[s][row][c]), summed in s order.
__global__ void reduce_partials_kernel(const float* __restrict__ part, int S, int rows, int R, ReduceOuts outs) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * R) return;
  const int row = idx / R, c = idx % R;
  float acc = 0.f;
  for (int s = 0; s < S; ++s) acc += part[(static_cast<size_t>(s) * rows + row) * R + c];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const ReduceOut& o = outs.o[j];
    if (o.ptr == nullptr || c < o.col0 || c >= o.col0 + 16) continue;
    const int cc = c - o.col0;
    const size_t off = o.transpose ? static_cast<size_t>(cc) * o.ld + row : static_cast<size_t>(row) * o.ld + cc;
    o.ptr[off] = __float2bfloat16_rn(o.scale * acc);
  }
}

// ---------------------------------------------------------------- launch --
static cudaError_t set_smem(const void* f, int bytes) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

cudaError_t launch_rowproj(int nv, const CUtensorMap& t, const CUtensorMap& v0, const CUtensorMap& v1, float* part,
                           int M, int K, int splits, int kb_per_split, int* status, cudaStream_t st) {
  const dim3 grid((M + 63) / 64, splits);
  if (nv == 1) {
    const int smem = SK_STAGES * (T_TILE + 2048) + 64 + 1024;
    cudaError_t e = set_smem((const void*)rowproj_kernel<1>, smem);
    if (e != cudaSuccess) return e;
    rowproj_kernel<1><<<grid, SK_THREADS, smem, st>>>(t, v0, v1, part, M, K, kb_per_split, status);
  } else {
    const int smem = SK_STAGES * (T_TILE + 4096) + 64 + 1024;
    cudaError_t e = set_smem((const void*)rowproj_kernel<2>, smem);
    if (e != cudaSuccess) return e;
    rowproj_kernel<2><<<grid, SK_THREADS, smem, st>>>(t, v0, v1, part, M, K, kb_per_split, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_colproj(int R, const CUtensorMap& t, const CUtensorMap& u, float* part, int M, int N, int splits,
                           int mb_per_split, int* status, cudaStream_t st) {
  const dim3 grid((N + 63) / 64, splits);
  const int smem = SK_STAGES * (T_TILE + 64 * R * 2) + 64 + 1024;
  if (R == 16) {
    cudaError_t e = set_smem((const void*)colproj_kernel<16>, smem);
    if (e != cudaSuccess) return e;
    colproj_kernel<16><<<grid, SK_THREADS, smem, st>>>(t, u, part, M, N, mb_per_split, status);
  } else {
    cudaError_t e = set_smem((const void*)colproj_kernel<32>, smem);
    if (e != cudaSuccess) return e;
    colproj_kernel<32><<<grid, SK_THREADS, smem, st>>>(t, u, part, M, N, mb_per_split, status);
  }
  return cudaGetLastError();
}

constexpr int DY_CC = 4;
cudaError_t launch_dypass(const CUtensorMap& t, const CUtensorMap& u, const CUtensorMap& b, float* gpart, float* qpart,
                          int M, int N, int rc_per_cta, int* status, cudaStream_t st) {
  const dim3 grid((N + DY_CC * 64 - 1) / (DY_CC * 64), (M + rc_per_cta * 64 - 1) / (rc_per_cta * 64));
  const int smem = SK_STAGES * (T_TILE + 2048 + 2048) + 64 + 1024;
  cudaError_t e = set_smem((const void*)dypass_kernel<DY_CC>, smem);
  if (e != cudaSuccess) return e;
  dypass_kernel<DY_CC><<<grid, SK_THREADS, smem, st>>>(t, u, b, gpart, qpart, M, N, rc_per_cta, status);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const float* part, int S, int rows, int R, const ReduceOuts& outs, cudaStream_t st) {
  const int n = rows * R;
  reduce_partials_kernel<<<(n + 255) / 256, 256, 0, st>>>(part, S, rows, R, outs);
  return cudaGetLastError();
}

}  // namespace ql
