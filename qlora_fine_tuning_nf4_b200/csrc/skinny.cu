// Rank-r ("skinny") products of the LoRA path on warp-level mma.sync.
//
// The Mistral blog ("用 Unsloth 微调 Mistral，速度提升 14 倍", item
// "10、11. 手动 Autograd") brackets every chained product so that the rank-r
// factor is contracted first; these kernels are those contractions:
//   rowproj   P[m, :]  = T[m, :] V          V = [K, 16*NV] (LoRA A)     X A, H A_d
//   colproj   Q[n, :]  = T[:, n]^T U        U = [M, R]                   X^T G (dA)
//   dypass    G[m, :]  = T[m, :] B^T  and  Q[n, :] = T[:, n]^T U          dY B^T, (X A)^T dY
// They are HBM-bound on T.  Each is persistent: its CTAs take equal
// contiguous ranges of the work units; one producer warp streams 64x64 bf16
// tiles of T (128B-swizzled) and the small factors through a 4-deep
// TMA/mbarrier ring, four consumer warps contract them (16 rows or columns of
// the tile each) and release each slot as soon as they are done with it.
// Every CTA writes one fp32 partial per output group it touched;
// `reduce_kernel` adds a group's partials in slot order, applies the LoRA
// scale and rounds to bf16, so results are deterministic.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cstring>


namespace ql {

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

// A rank-side factor tile: 64 rows x W bf16 columns, stored as W / SUBW
// sub-tiles of SUBW = min(W, 64) columns, each in the TMA swizzle of its row
// width (32, 64 or 128 bytes) so that 8-row ldmatrix phases hit distinct banks.
template <int W>
struct FTile {
  static constexpr int SUBW = W < 64 ? W : 64;
  static constexpr int ROWB = SUBW * 2;
  static constexpr int SUB_BYTES = 64 * ROWB;
  static constexpr int BYTES = (W / SUBW) * SUB_BYTES;
  // byte offset of the 16-byte chunk holding columns [c, c + 8) of row k
  QL_DEV static int off(int k, int c) {
    const int x = ROWB == 128 ? (k & 7) : (ROWB == 64 ? ((k >> 1) & 3) : ((k >> 2) & 1));
    return (c / SUBW) * SUB_BYTES + k * ROWB + ((((c % SUBW) >> 3) ^ x) << 4);
  }
};
// B-fragment (16x8) of a factor tile used as [k][n]: rows [k0, k0+16), columns [n0, n0+8).
template <int W>
QL_DEV void frag_b_kn_f(uint32_t tile, int k0, int n0, int lane, uint32_t (&b)[2]) {
  ldsm_x2_t(tile + FTile<W>::off(k0 + (lane & 15), n0), b[0], b[1]);
}
// B-fragment from a 128B-swizzled [n][k] tile (rows = output column n,
// 128 bytes of k per row): reduction [k0, k0+16), columns [n0, n0+8).
QL_DEV void frag_b_nk(uint32_t tile, int k0, int n0, int lane, uint32_t (&b)[2]) {
  const int n = n0 + (lane & 7);
  const int chunk = (k0 >> 3) + ((lane >> 3) & 1);
  ldsm_x2(tile + n * 128 + ((chunk ^ (n & 7)) << 4), b[0], b[1]);
}

// ------------------------------------------------------------ pipeline ---
constexpr int SK_CWARPS = 4;                         // consumer warps
constexpr int SK_THREADS = 32 * (SK_CWARPS + 1);     // + the producer warp
constexpr int SK_STAGES = 4;                         // 4 CTAs per SM: 16 consumer warps

QL_DEV uint32_t sk_full(uint32_t bars, int s) { return bars + 8u * s; }
QL_DEV uint32_t sk_empty(uint32_t bars, int s) { return bars + 8u * (SK_STAGES + s); }

QL_DEV void sk_init(uint32_t bars) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(sk_full(bars, s), 1);
      mbar_init(sk_empty(bars, s), SK_CWARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
}

// Test-only fault injection (qlora_test_inject_timeout): when set, the first
// CTA of the next skinny launch leaves its tile 1 unloaded, so that CTA's
// consumers run into their bounded wait; the launch clears it (one shot).
__device__ int g_inject_timeout = 0;

// Producer (one thread): issue(i, s, full_bar) loads tile i of the CTA's range
// into slot s once the consumers released it; afterwards waits (bounded, and
// after an error too) until every load it issued has landed, so no copy is in
// flight when the CTA exits.
template <typename Issue>
QL_DEV void sk_produce(int ntiles, uint32_t bars, int* status, Issue issue) {
  int skip = -1;
  if (blockIdx.x == 0 && ntiles > 1 && atomicExch(&g_inject_timeout, 0) != 0) skip = 1;
  int i = 0;
  for (; i < ntiles; ++i) {
    const int s = i % SK_STAGES;
    if (!mbar_wait(sk_empty(bars, s), ((i / SK_STAGES) & 1) ^ 1, status)) break;
    if (i != skip) issue(i, s, sk_full(bars, s));
  }
  for (int j = i > SK_STAGES ? i - SK_STAGES : 0; j < i; ++j)
    if (j != skip) mbar_drain(sk_full(bars, j % SK_STAGES), (j / SK_STAGES) & 1);
}

// Consumer side of tile i: wait until it has landed (uniform over the warp).
// After a failed wait the warp stops waiting (the status word holds the
// timeout) and walks the rest of its tiles without touching them.
QL_DEV bool sk_acquire(uint32_t bars, int i, bool ok, int* status) {
  return ok && __all_sync(0xffffffffu, mbar_wait(sk_full(bars, i % SK_STAGES), (i / SK_STAGES) & 1, status));
}
// ... and hand the slot back (the fragments read from it are consumed by then).
QL_DEV void sk_release(uint32_t bars, int i, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(sk_empty(bars, i % SK_STAGES));
}

// Tile range [t0, t1) of CTA c.
QL_DEV void sk_range(const SkPart& sp, int units, int c, int& t0, int& t1) {
  t0 = part_begin(c, sp.U, sp.P) * sp.align;
  t1 = min(part_begin(c + 1, sp.U, sp.P) * sp.align, units);
}

// Store a warp's 16 x (8 * NB) accumulator block (mma C layout) at rows
// [r0, r0 + 16) of a row-major fp32 [rows][ld] array, then clear it.
template <int NB>
QL_DEV void store_acc(float* base, int ld, int r0, int lane, float (&acc)[NB][4]) {
  const int r = r0 + (lane >> 2);
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int c = nb * 8 + (lane & 3) * 2;
    *reinterpret_cast<float2*>(base + static_cast<size_t>(r) * ld + c) = make_float2(acc[nb][0], acc[nb][1]);
    *reinterpret_cast<float2*>(base + static_cast<size_t>(r + 8) * ld + c) = make_float2(acc[nb][2], acc[nb][3]);
    acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
  }
}

// ------------------------------------------------------------- rowproj ---
// Units: 64x64 tiles (rc, kc), kc fastest; group = row block rc (nkc units).
// job.part[rc][slot][64][NF * RW]: T V over the CTA's tiles of row block rc,
// V = NF factors of RW columns side by side.  BT: the single factor is given
// transposed, as the LoRA right factor B [RW, K] (G = T B^T).
template <int RW, int NF, bool BT>
__global__ void __launch_bounds__(SK_THREADS) rowproj_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                             const __grid_constant__ CUtensorMap tmap_v0,
                                                             const __grid_constant__ CUtensorMap tmap_v1,
                                                             const __grid_constant__ CUtensorMap tmap_v2,
                                                             const __grid_constant__ ReduceJob job, int nkc,
                                                             int* status) {
  using F = FTile<RW>;
  constexpr int R = NF * RW;
  constexpr int V_TILE = BT ? RW * 128 : F::BYTES;
  constexpr int STAGE = T_TILE + NF * V_TILE;
  static_assert(!BT || NF == 1, "transposed factor: one factor");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  int t0, t1;
  sk_range(job.sp, job.groups * nkc, c, t0, t1);
  const int nt = t1 - t0;
  sk_init(bars);

  if (warp == SK_CWARPS) {
    if (lane == 0)
      sk_produce(nt, bars, status, [&](int i, int s, uint32_t fb) {
        const int t = t0 + i, rc = t / nkc, kc = t % nkc;
        const uint32_t st = sbase + s * STAGE;
        mbar_arrive_expect_tx(fb, STAGE);
        tma_load_2d(st, &tmap_t, fb, kc * 64, rc * 64);
        if (BT) {
          tma_load_2d(st + T_TILE, &tmap_v0, fb, kc * 64, 0);
        } else {
#pragma unroll
          for (int f = 0; f < NF; ++f)
#pragma unroll
            for (int sub = 0; sub < RW / F::SUBW; ++sub)
              tma_load_2d(st + T_TILE + f * V_TILE + sub * F::SUB_BYTES,
                          f == 0 ? &tmap_v0 : (f == 1 ? &tmap_v1 : &tmap_v2), fb, sub * F::SUBW, kc * 64);
        }
      });
    return;
  }
  float acc[R / 8][4] = {};
  bool ok = true;
  for (int i = 0; i < nt; ++i) {
    const int t = t0 + i, rc = t / nkc, kc = t % nkc;
    ok = sk_acquire(bars, i, ok, status);
    if (ok) {
      const uint32_t tb = sbase + (i % SK_STAGES) * STAGE;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        frag_a_rows(tb, warp * 16, kk * 16, lane, a);
#pragma unroll
        for (int nb = 0; nb < R / 8; ++nb) {
          uint32_t b[2];
          if (BT)
            frag_b_nk(tb + T_TILE, kk * 16, nb * 8, lane, b);
          else
            frag_b_kn_f<RW>(tb + T_TILE + (nb / (RW / 8)) * V_TILE, kk * 16, (nb % (RW / 8)) * 8, lane, b);
          mma_bf16_16816(acc[nb], a[0], a[1], a[2], a[3], b[0], b[1]);
        }
      }
      sk_release(bars, i, lane);
    }
    if (kc == nkc - 1 || i == nt - 1) {
      const int slot = c - sk_first(job.sp, rc);
      if (dev_check(rc < job.groups && slot >= 0 && slot < job.slot_cap, status))
        store_acc(job.part + static_cast<size_t>(rc * job.slot_cap + slot) * 64 * R, R, warp * 16, lane, acc);
    }
  }
}

// ------------------------------------------------------------- colproj ---
// Units: (cb, mc) = 64 rows x CC column chunks of 64, mc fastest; group =
// column block cb (CC * 64 columns, nmc units).  A unit's chunks are 64x64
// tiles of T, one ring stage each, side by side in the same 64 rows, so a CTA
// walking down its column block reads CC * 128 contiguous bytes of every row;
// each stage also carries the unit's U rows (from L2).
// job.part[cb][slot][CC * 64][R]: T^T U over the CTA's rows of column block cb.
// CC is 1 or, for wide operands (chosen on the host), colproj_cc(R): the
// accumulators then hold CC * R / 2 floats per thread, at most 64.
constexpr int colproj_cc(int R) { return R <= 32 ? 4 : (R == 64 ? 2 : 1); }
int colproj_chunks(int R) { return colproj_cc(R); }
template <int R, int CC>
__global__ void __launch_bounds__(SK_THREADS) colproj_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                             const __grid_constant__ CUtensorMap tmap_u,
                                                             const __grid_constant__ ReduceJob job, int nmc,
                                                             int nch, int* status) {
  using F = FTile<R>;
  constexpr int STAGE = T_TILE + F::BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  int u0, u1;
  sk_range(job.sp, job.groups * nmc, c, u0, u1);
  auto chunks = [&](int cb) { return min(CC, nch - cb * CC); };
  int nt = 0;
  for (int u = u0; u < u1; ++u) nt += chunks(u / nmc);
  sk_init(bars);

  if (warp == SK_CWARPS) {
    if (lane == 0) {
      int u = u0, cc = 0;
      sk_produce(nt, bars, status, [&](int, int s, uint32_t fb) {
        const int cb = u / nmc, mc = u % nmc;
        const uint32_t st = sbase + s * STAGE;
        mbar_arrive_expect_tx(fb, STAGE);
        tma_load_2d(st, &tmap_t, fb, (cb * CC + cc) * 64, mc * 64);
#pragma unroll
        for (int sub = 0; sub < R / F::SUBW; ++sub)
          tma_load_2d(st + T_TILE + sub * F::SUB_BYTES, &tmap_u, fb, sub * F::SUBW, mc * 64);
        if (++cc == chunks(cb)) {
          cc = 0;
          ++u;
        }
      });
    }
    return;
  }
  float acc[CC][R / 8][4] = {};
  int i = 0;
  bool ok = true;
  for (int u = u0; u < u1; ++u) {
    const int cb = u / nmc, ncc = chunks(cb);
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) {
      if (cc >= ncc) break;
      ok = sk_acquire(bars, i, ok, status);
      if (ok) {
        const uint32_t tb = sbase + (i % SK_STAGES) * STAGE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a[4];
          frag_a_cols(tb, kk * 16, warp * 16, lane, a);
#pragma unroll
          for (int nb = 0; nb < R / 8; ++nb) {
            uint32_t b[2];
            frag_b_kn_f<R>(tb + T_TILE, kk * 16, nb * 8, lane, b);
            mma_bf16_16816(acc[cc][nb], a[0], a[1], a[2], a[3], b[0], b[1]);
          }
        }
        sk_release(bars, i, lane);
      }
      ++i;
    }
    if (u == u1 - 1 || (u + 1) / nmc != cb) {
      const int slot = c - sk_first(job.sp, cb);
      float* qb = job.part + static_cast<size_t>(cb * job.slot_cap + slot) * (CC * 64) * R;
      if (dev_check(cb < job.groups && slot >= 0 && slot < job.slot_cap, status)) {
#pragma unroll
        for (int q = 0; q < CC; ++q) store_acc(qb + q * 64 * R, R, warp * 16, lane, acc[q]);
      }
    }
  }
}

// -------------------------------------------------------------- dypass ---
// One read of T = dY [M, N] gives both
//   G[m, :] = sum_n T[m,n] Bl[:, n]   (Bl = LoRA B, [16, N])
//   Q[n, :] = sum_m T[m,n] U[m, :]    (U = X A, [M, 16])
// Units: (cb, rc) = 64 rows x DY_CC column chunks of 64, rc fastest.
//   gjob.part[rc][cb][64][16]: G over the unit's columns (one writer per unit);
//   qjob.part[cb][slot][DY_CC * 64][16]: Q of column block cb over the CTA's rows.
constexpr int DY_CC = 4;
__global__ void __launch_bounds__(SK_THREADS) dypass_kernel(const __grid_constant__ CUtensorMap tmap_t,
                                                            const __grid_constant__ CUtensorMap tmap_u,
                                                            const __grid_constant__ CUtensorMap tmap_b,
                                                            const __grid_constant__ ReduceJob gjob,
                                                            const __grid_constant__ ReduceJob qjob, int nch,
                                                            int* status) {
  constexpr int CC = DY_CC;
  constexpr int U_TILE = 64 * 16 * 2;
  constexpr int B_TILE = 16 * 64 * 2;
  constexpr int STAGE = T_TILE + U_TILE + B_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bars = sbase + SK_STAGES * STAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int nrc = gjob.groups, ncb = qjob.groups;
  const SkPart& sp = qjob.sp;
  int u0, u1;
  sk_range(sp, ncb * nrc, c, u0, u1);
  auto chunks = [&](int cb) { return min(CC, nch - cb * CC); };
  int nt = 0;
  for (int u = u0; u < u1; ++u) nt += chunks(u / nrc);
  sk_init(bars);

  if (warp == SK_CWARPS) {
    if (lane == 0) {
      int u = u0, cc = 0;
      sk_produce(nt, bars, status, [&](int, int s, uint32_t fb) {
        const int cb = u / nrc, rc = u % nrc, col = (cb * CC + cc) * 64;
        const uint32_t st = sbase + s * STAGE;
        mbar_arrive_expect_tx(fb, STAGE);
        tma_load_2d(st, &tmap_t, fb, col, rc * 64);
        tma_load_2d(st + T_TILE, &tmap_u, fb, 0, rc * 64);
        tma_load_2d(st + T_TILE + U_TILE, &tmap_b, fb, col, 0);
        if (++cc == chunks(cb)) {
          cc = 0;
          ++u;
        }
      });
    }
    return;
  }
  float qacc[CC][2][4] = {};
  int i = 0;
  bool ok = true;
  for (int u = u0; u < u1; ++u) {
    const int cb = u / nrc, rc = u % nrc, ncc = chunks(cb);
    float gacc[2][4] = {};
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) {
      if (cc >= ncc) break;
      ok = sk_acquire(bars, i, ok, status);
      if (ok) {
        const uint32_t tb = sbase + (i % SK_STAGES) * STAGE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a[4];
          // G += T[rows 16w.., cols kk*16..] * Bl^T
          frag_a_rows(tb, warp * 16, kk * 16, lane, a);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            uint32_t b[2];
            frag_b_nk(tb + T_TILE + U_TILE, kk * 16, nb * 8, lane, b);
            mma_bf16_16816(gacc[nb], a[0], a[1], a[2], a[3], b[0], b[1]);
          }
          // Q += T[rows kk*16.., cols 16w..]^T * U
          frag_a_cols(tb, kk * 16, warp * 16, lane, a);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            uint32_t b[2];
            frag_b_kn_f<16>(tb + T_TILE, kk * 16, nb * 8, lane, b);
            mma_bf16_16816(qacc[cc][nb], a[0], a[1], a[2], a[3], b[0], b[1]);
          }
        }
        sk_release(bars, i, lane);
      }
      ++i;
    }
    if (dev_check(rc < nrc && cb < gjob.slot_cap, status))
      store_acc(gjob.part + static_cast<size_t>(rc * ncb + cb) * 64 * 16, 16, warp * 16, lane, gacc);
    if (u == u1 - 1 || (u + 1) / nrc != cb) {
      const int slot = c - sk_first(sp, cb);
      float* qb = qjob.part + static_cast<size_t>(cb * qjob.slot_cap + slot) * (CC * 64) * 16;
      if (dev_check(cb < ncb && slot >= 0 && slot < qjob.slot_cap, status)) {
#pragma unroll
        for (int q = 0; q < CC; ++q) store_acc(qb + q * 64 * 16, 16, warp * 16, lane, qacc[q]);
      }
    }
  }
}

// ------------------------------------------------------------- reduce ----
// out = bf16(scale * sum over the group's slots of part), summed in slot
// order.  One thread per four consecutive partial columns; its slot loads are
// issued sixteen at a time.  One launch serves up to kMaxReduceJobs
// reductions (each with its own partial region): job k takes the threads
// [start[k], start[k + 1]).
struct ReduceJobs {
  ReduceJob j[kMaxReduceJobs];
  int start[kMaxReduceJobs + 1];  // prefix sums of rows * R / 4 (float4 elements)
  int n;                          // jobs in use
};
__global__ void __launch_bounds__(256) reduce_kernel(const __grid_constant__ ReduceJobs js) {
  grid_dep_wait();
  grid_dep_launch();
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= js.start[js.n]) return;
  int k = 0;
  while (k + 1 < js.n && idx >= js.start[k + 1]) ++k;
  idx -= js.start[k];
  const ReduceJob& j = js.j[k];
  const int row = (idx * 4) / j.R, c = (idx * 4) % j.R;
  const int g = row / j.grows, r = row % j.grows;
  int ns = j.nslots > 0 ? j.nslots : sk_slots(j.sp, g);
  if (!dev_check(g < j.groups && ns <= j.slot_cap, j.status)) ns = g < j.groups ? j.slot_cap : 0;
  const size_t slot_stride = static_cast<size_t>(j.grows) * j.R;
  const float* p = j.part + static_cast<size_t>(g) * j.slot_cap * slot_stride + static_cast<size_t>(r) * j.R + c;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < ns; s += 16) {
    float4 v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t)
      if (s + t < ns) v[t] = __ldg(reinterpret_cast<const float4*>(p + (s + t) * slot_stride));
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (s + t < ns) {
        acc.x += v[t].x;
        acc.y += v[t].y;
        acc.z += v[t].z;
        acc.w += v[t].w;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const ReduceOut& o = j.outs.o[q];
    if (o.ptr == nullptr || c < o.col0 || c >= o.col0 + o.width) continue;
    const int cc = c - o.col0;
    const bf16 b0 = __float2bfloat16_rn(o.scale * acc.x), b1 = __float2bfloat16_rn(o.scale * acc.y);
    const bf16 b2 = __float2bfloat16_rn(o.scale * acc.z), b3 = __float2bfloat16_rn(o.scale * acc.w);
    if (o.transpose) {
      bf16* d = o.ptr + static_cast<size_t>(cc) * o.ld + row;
      d[0] = b0;
      d[o.ld] = b1;
      d[2 * static_cast<size_t>(o.ld)] = b2;
      d[3 * static_cast<size_t>(o.ld)] = b3;
    } else {
      __nv_bfloat162 lo, hi;
      lo.x = b0;
      lo.y = b1;
      hi.x = b2;
      hi.y = b3;
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(o.ptr + static_cast<size_t>(row) * o.ld + cc) = w;
    }
  }
}

// ---------------------------------------------------------------- launch --
static cudaError_t set_smem(const void* f, int bytes) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}
static int sk_smem(int stage) { return SK_STAGES * stage + 2 * SK_STAGES * 8 + 1024; }

template <int RW, int NF, bool BT>
static cudaError_t launch_rowproj_t(const CUtensorMap& t, const CUtensorMap& v0, const CUtensorMap& v1,
                                    const CUtensorMap& v2, const ReduceJob& job, int nkc, int* status,
                                    cudaStream_t st) {
  const int vt = BT ? RW * 128 : FTile<RW>::BYTES;
  const int smem = sk_smem(T_TILE + NF * vt);
  auto k = rowproj_kernel<RW, NF, BT>;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(job.sp.P), dim3(SK_THREADS), smem, st, t, v0, v1, v2, job, nkc, status);
}

// rank rw in {16, 32, 64}; nf factors (1 to 3), or bt: one factor given as B [rw, K]
cudaError_t launch_rowproj(int rw, int nf, bool bt, const CUtensorMap& t, const CUtensorMap& v0,
                           const CUtensorMap& v1, const CUtensorMap& v2, const ReduceJob& job, int nkc, int* status,
                           cudaStream_t st) {
#define QL_ROW(RW_)                                                                              \
  if (rw == RW_) {                                                                               \
    if (bt) return launch_rowproj_t<RW_, 1, true>(t, v0, v1, v2, job, nkc, status, st);          \
    if (nf == 1) return launch_rowproj_t<RW_, 1, false>(t, v0, v1, v2, job, nkc, status, st);    \
    if (nf == 2) return launch_rowproj_t<RW_, 2, false>(t, v0, v1, v2, job, nkc, status, st);    \
    return launch_rowproj_t<RW_, 3, false>(t, v0, v1, v2, job, nkc, status, st);                 \
  }
  QL_ROW(16)
  QL_ROW(32)
  QL_ROW(64)
#undef QL_ROW
  return cudaErrorInvalidValue;
}

template <int R, int CC>
static cudaError_t launch_colproj_t(const CUtensorMap& t, const CUtensorMap& u, const ReduceJob& job, int nmc,
                                    int nch, int* status, cudaStream_t st) {
  const int smem = sk_smem(T_TILE + FTile<R>::BYTES);
  auto k = colproj_kernel<R, CC>;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(job.sp.P), dim3(SK_THREADS), smem, st, t, u, job, nmc, nch, status);
}

// R in {16, 32, 64, 128}; cc = 1 or colproj_cc(R) column chunks per unit; nch = column chunks of 64 in T
cudaError_t launch_colproj(int R, int cc, const CUtensorMap& t, const CUtensorMap& u, const ReduceJob& job, int nmc,
                           int nch, int* status, cudaStream_t st) {
#define QL_COL(R_)                                                                              \
  if (R == R_) {                                                                                \
    if (cc == 1) return launch_colproj_t<R_, 1>(t, u, job, nmc, nch, status, st);               \
    if (cc == colproj_cc(R_)) return launch_colproj_t<R_, colproj_cc(R_)>(t, u, job, nmc, nch, status, st); \
    return cudaErrorInvalidValue;                                                               \
  }
  QL_COL(16)
  QL_COL(32)
  QL_COL(64)
  QL_COL(128)
#undef QL_COL
  return cudaErrorInvalidValue;
}

cudaError_t launch_dypass(const CUtensorMap& t, const CUtensorMap& u, const CUtensorMap& b, const ReduceJob& gjob,
                          const ReduceJob& qjob, int nch, int* status, cudaStream_t st) {
  const int smem = sk_smem(T_TILE + 2048 + 2048);
  cudaError_t e = set_smem((const void*)dypass_kernel, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(dypass_kernel, dim3(qjob.sp.P), dim3(SK_THREADS), smem, st, t, u, b, gjob, qjob, nch, status);
}

cudaError_t arm_inject_timeout() {
  const int one = 1;
  return cudaMemcpyToSymbol(g_inject_timeout, &one, sizeof(one));
}

// One launch for `n` reductions (1 <= n <= kMaxReduceJobs).
cudaError_t launch_reduce(const ReduceJob* jobs, int n, cudaStream_t st) {
  if (n < 1 || n > kMaxReduceJobs) return cudaErrorInvalidValue;
  ReduceJobs js;
  std::memset(&js, 0, sizeof(js));
  js.n = n;
  int64_t total = 0;
  for (int k = 0; k < n; ++k) {
    js.j[k] = jobs[k];
    js.start[k] = static_cast<int>(total);
    total += static_cast<int64_t>(jobs[k].rows) * jobs[k].R / 4;
  }
  if (total >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  js.start[n] = static_cast<int>(total);
  if (total == 0) return cudaSuccess;
  return launch_pdl(reduce_kernel, dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256), 0, st, js);
}

}  // namespace ql
