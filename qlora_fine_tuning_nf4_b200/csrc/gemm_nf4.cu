// NF4 x bf16 tensor-core GEMM for sm_100a with the frozen weight dequantised
// into shared memory inside the mainloop, the LoRA term as extra K=16 MMAs
// into the same TMEM accumulator, and fused gated-activation epilogues.
//
// What it computes (Mistral blog "用 Unsloth 微调 Mistral，速度提升 14 倍",
// items "2. Bitsandbytes bfloat16" and "10、11. 手动 Autograd"; Gemma blog
// section "GeGLU 与 Swiglu 激活函数"):
//   forward   Y  = X  dequant(W)^T + (s X A) B            (MODE_FWD)
//   gate/up   e, g as above; h = act(e) g                  (MODE_FWD_GLU)
//   backward  dX = dY dequant(W)   + (s dY B^T) A^T        (MODE_BWD)
//   down bwd  dH as above; dE = dH g act'(e), dG = dH act(e) (EPI_GLU_BWD)
// Two ways to feed the B operand (the weight), chosen per launch:
//  * in-mainloop dequantisation: the dequantised weight never exists in HBM;
//    each CTA expands the NF4 codes of its B tile straight to bf16 in shared
//    memory, k-block by k-block, while the tensor cores consume earlier ones;
//  * staged: the caller has expanded the whole weight once into a bf16 buffer
//    (the HBM-bound dequantisation kernel) and the B tiles arrive by TMA like
//    the A tiles.  Every B tile is then decoded once per call instead of once
//    per output-row tile, and the shared-memory stores of the decoded tile
//    leave the mainloop.
//
// Structure (persistent; one output tile at a time per CTA, or per CTA pair
// with cta_group::2):
//   warp 0       TMA producer: A tiles (and staged B tiles), LoRA operands
//   warp 1       TMEM allocation; lane 0 of the leader CTA issues tcgen05.mma
//   warp 2       raw NF4 codes + absmax by TMA (in-mainloop feed only)
//   warps 3-10   epilogue: TMEM -> registers -> activation -> global
//   warps 11-18  dequantisers: raw codes -> bf16 B tile (in-mainloop feed only)
// Pipelines: raw ring (TMA -> dequantisers), operand ring (A by TMA, B by the
// dequantisers or by TMA -> MMA), two accumulators (MMA -> epilogue).
#include "kernels.cuh"
#include "ptx.cuh"

namespace ql {

// NF4 levels (QLoRA NormalFloat construction, binary32), as bit patterns.
__device__ __forceinline__ float nf4_level(int i) {
  constexpr uint32_t kBits[16] = {0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
                                  0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
                                  0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};
  return __uint_as_float(kBits[i]);
}

// Per-block product table T[q] = bf16(level[q] * absmax), split into the low
// bytes (tl) and high bytes (th) of the 16 bf16 values, 4 per register.
QL_DEV void nf4_block_table(float absmax, uint32_t (&tl)[4], uint32_t (&th)[4]) {
  uint32_t p[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) p[k] = pack_bf16x2(nf4_level(2 * k) * absmax, nf4_level(2 * k + 1) * absmax);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    tl[k] = prmt(p[2 * k], p[2 * k + 1], 0x6420u);
    th[k] = prmt(p[2 * k], p[2 * k + 1], 0x7531u);
  }
}

// Eight 4-bit codes (one 32-bit word; byte b holds element 2b in its high
// nibble and 2b+1 in its low nibble) -> eight bf16 in element order.
// Byte-permute lookups: the low three bits of each nibble index an 8-entry
// half of the table; bit 3 chooses the half through a sign-replicated mask.
QL_DEV uint4 nf4_decode8(uint32_t w, const uint32_t (&tl)[4], const uint32_t (&th)[4]) {
  const uint32_t sel = w & 0x77777777u;
  const uint32_t sel_hi = sel >> 16;
  const uint32_t w4 = w << 4;
  const uint32_t m_lo = prmt(w, w4, 0x9D8Cu);
  const uint32_t m_hi = prmt(w, w4, 0xBFAEu);
  uint4 out;
  uint32_t L = (prmt(tl[0], tl[1], sel) & ~m_lo) | (prmt(tl[2], tl[3], sel) & m_lo);
  uint32_t H = (prmt(th[0], th[1], sel) & ~m_lo) | (prmt(th[2], th[3], sel) & m_lo);
  out.x = prmt(L, H, 0x4051u);
  out.y = prmt(L, H, 0x6273u);
  L = (prmt(tl[0], tl[1], sel_hi) & ~m_hi) | (prmt(tl[2], tl[3], sel_hi) & m_hi);
  H = (prmt(th[0], th[1], sel_hi) & ~m_hi) | (prmt(th[2], th[3], sel_hi) & m_hi);
  out.z = prmt(L, H, 0x4051u);
  out.w = prmt(L, H, 0x6273u);
  return out;
}

// Activations in fp32 on the hardware's approximate exp2 / divide / tanh units
// (relative error well below the bf16 rounding of the stored results).  Under
// the power cap every epilogue instruction costs step time: the approximate
// divide instead of a correctly rounded reciprocal made the MLP step ~0.8% faster.
QL_DEV float fast_sigmoid(float e) { return __fdividef(1.0f, 1.0f + __expf(-e)); }
QL_DEV float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
QL_DEV float act_f(int act, float e) {
  if (act == ACT_SILU) return e * fast_sigmoid(e);
  const float t = tanh_approx(0.7978845608028654f * (e + 0.044715f * e * e * e));
  return 0.5f * e * (1.0f + t);
}
// (act(e), act'(e))
QL_DEV void act_fg(int act, float e, float& f, float& g) {
  if (act == ACT_SILU) {
    const float s = fast_sigmoid(e);
    f = e * s;
    g = s * (1.0f + e * (1.0f - s));
  } else {
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    const float t = tanh_approx(k0 * (e + k1 * e * e * e));
    f = 0.5f * e * (1.0f + t);
    g = 0.5f * (1.0f + t) + 0.5f * e * (1.0f - t * t) * k0 * (1.0f + 3.0f * k1 * e * e);
  }
}

// Tile configuration.  A CTA owns MH accumulators of 128 rows (TMEM lanes) x
// BNT columns; with cta_group::2 a pair of CTAs issues each MMA with M = 256
// and each CTA supplies BNC = BNT / 2 columns of the dequantised B operand.
//   (CG, MH) = (1, 1): 128 x 256 per CTA
//   (CG, MH) = (2, 1): 256 x 256 per pair
//   (CG, MH) = (2, 2): 512 x 128 per pair -- each dequantised B tile feeds two
//                      M = 256 MMAs, halving the dequantisation per MMA.
template <int MODE, int CG, int MH, bool ST>
struct GemmCfg {
  static constexpr int BM = 128;                 // rows per CTA per M-half (TMEM lanes)
  static constexpr int BNT = 256 / MH;           // MMA N (whole pair)
  static constexpr int BNC = BNT / CG;           // B columns produced per CTA
  static constexpr int BK = 64;                  // reduction block (one NF4 block, one 128B row)
  static constexpr int NB = BNC;                 // NF4 blocks dequantised per CTA per k-block
  static constexpr int BOXR = BNC < 128 ? BNC : 128;  // rows per TMA box of codes / absmax / LoRA rows
  static constexpr int A_TILE = BM * BK * 2;
  static constexpr int A_BYTES = MH * A_TILE;
  static constexpr int B_BYTES = BNC * BK * 2;
  static constexpr int RC_BYTES = NB * 32;
  static constexpr int RA_BYTES = (MODE == MODE_BWD) ? 64 * 16 : BNC * 16;
  static constexpr int S = ST ? 5 : ((CG == 1) ? 3 : (MH == 1 ? 5 : 4));  // operand stages
  static constexpr int RS = ST ? 0 : ((CG == 1) ? 4 : (MH == 1 ? 6 : 8));  // raw stages
  // dedicated LoRA operand tiles (rank 16) of the in-mainloop feed; the staged
  // feed streams its LoRA operands through the operand ring instead
  static constexpr int LA_BYTES = ST ? 0 : BM * 16 * 2;  // one LoRA left operand tile (128 rows x 16)
  static constexpr int LBOP = ST ? 0 : BNC * 32;         // one LoRA right operand (BNC x 16 bf16)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + S * A_BYTES;
  static constexpr int OFF_RC = OFF_B + S * B_BYTES;
  static constexpr int OFF_RA = OFF_RC + RS * RC_BYTES;
  static constexpr int OFF_LA = OFF_RA + RS * RA_BYTES;
  static constexpr int OFF_LB = OFF_LA + MH * 2 * LA_BYTES;
  static constexpr int OFF_EPI = OFF_LB + 2 * LBOP;
  // staged feed: per epilogue warp three 32 x 32 bf16 output slots (64B-swizzled) for TMA stores
  static constexpr int EPI_SLOT = 32 * 32 * 2;
  static constexpr int EPI_BYTES = ST ? 8 * 3 * EPI_SLOT : 0;
  static constexpr int OFF_BAR = OFF_EPI + EPI_BYTES;
  static constexpr int NBAR = 2 * S + 2 * RS + 7;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  static constexpr int EPI_WARPS = 8;            // two per TMEM lane quadrant
  static constexpr int DQ_WARPS = ST ? 0 : 8;
  static constexpr int EPI_WARP0 = 3;            // warps 0: A/LoRA TMA, 1: MMA, 2: raw-code TMA
  static constexpr int DQ_WARP0 = EPI_WARP0 + EPI_WARPS;
  static constexpr int THREADS = (DQ_WARP0 + DQ_WARPS) * 32;
  static constexpr int TMEM_COLS = 512;          // two accumulators of MH x BNT = 256 columns
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_LA % 1024 == 0 && OFF_RA % 1024 == 0 && OFF_LB % 1024 == 0 && OFF_EPI % 1024 == 0,
                "1024B alignment");
  static_assert(256 % NB == 0 && NB % 64 == 0, "dequantiser mapping");
};

// Roles: warp 0 issues the TMA loads of the A operand and the LoRA operands,
// warp 1 allocates TMEM and (leader CTA, one thread) issues tcgen05.mma,
// warp 2 streams the raw NF4 codes + absmax, running up to RS k-blocks ahead
// of the dequantisers independently of the MMA's progress, warps 3-10 drain
// the accumulators (epilogue), warps 11-18 dequantise.
//
// Persistent kernel: each CTA (or CTA pair) walks the output tiles
// t = cluster, cluster + clusters, ... (N tiles fastest).  Every role iterates
// the same tile sequence; j counts 64-wide reduction blocks across tiles and
// indexes the rings, so barrier phases follow from j and the tile counter.
template <int MODE, int EPI, int CG, int MH, bool ST>
__global__ void __launch_bounds__(GemmCfg<MODE, CG, MH, ST>::THREADS, 1)
    gemm_nf4_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs args) {
  using C = GemmCfg<MODE, CG, MH, ST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;

  const int bn_out = (EPI == EPI_GLU_FWD) ? C::BNT / 2 : C::BNT;  // output columns per tile
  const int bm_pair = C::BM * CG * MH;                            // output rows per tile
  const int n_tiles = (args.N + bn_out - 1) / bn_out;
  const int m_tiles = (args.M + bm_pair - 1) / bm_pair;
  const int total_tiles = n_tiles * m_tiles;
  const int cluster = blockIdx.x / CG;
  const int clusters = gridDim.x / CG;
  const int nk = args.nkb0 + args.nkb1;
  // Checked build: the arguments the tile walk and the rings depend on.  They are
  // the same for every CTA, so on failure the whole grid leaves here, before any
  // barrier, TMEM or cluster operation.
  if (!dev_check(args.M > 0 && args.N > 0 && args.nkb0 > 0 && args.nkb1 >= 0 && args.group_m >= 1 &&
                     args.lora >= 0 && args.lora <= (ST ? 3 : 2) && args.ldo >= args.N &&
                     (!ST || args.lora == 0 || (args.lora_k16 >= 1 && args.lora_k16 <= 4)),
                 args.status)) {
    grid_dep_wait();
    return;
  }

  // barriers
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::S + s); };
  auto rfull_bar = [&](int s) { return bar0 + 8u * (2 * C::S + s); };
  auto rempty_bar = [&](int s) { return bar0 + 8u * (2 * C::S + C::RS + s); };
  const uint32_t lora_full = bar0 + 8u * (2 * C::S + 2 * C::RS);
  const uint32_t lora_empty = lora_full + 8u;
  const uint32_t acc_full0 = lora_full + 16u;   // [2]
  const uint32_t acc_empty0 = lora_full + 32u;  // [2]
  const uint32_t drain_bar = lora_full + 48u;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + C::NBAR * 8);

  // Gated forward: the pair tile's B columns are [gate | up].  LoRA operand i
  // (0 = gate, 1 = up) is loaded into the 64-column chunks of this CTA that
  // belong to it; the other chunks stay zero, so both LoRA MMAs span all BNT
  // columns and each only adds to its own half.
  auto glu_chunk_is_gate = [&](int c) { return static_cast<int>(rank) * C::BNC + c * 64 < C::BNT / 2; };
  if (!ST && EPI == EPI_GLU_FWD) {
    for (int c = 0; c < C::BNC / 64; ++c) {
      const int zero_op = glu_chunk_is_gate(c) ? 1 : 0;
      uint4* z = reinterpret_cast<uint4*>(sgen + C::OFF_LB + zero_op * C::LBOP + c * 2048);
      for (int i = threadIdx.x; i < 2048 / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      mbar_init(full_bar(s), ST ? 1 : 1 + CG * (C::NB / 32));
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < C::RS; ++s) {
      mbar_init(rfull_bar(s), 1);
      mbar_init(rempty_bar(s), C::NB / 32);
    }
    mbar_init(lora_full, 1);
    mbar_init(lora_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full0 + 8u * b, 1);
      mbar_init(acc_empty0 + 8u * b, CG * C::EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<CG>(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish<CG>();
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  grid_dep_wait();  // the previous kernel's outputs (this kernel's inputs) are complete
  grid_dep_launch();

  // shared::cluster address of a barrier in the pair's leader CTA
  auto leader = [&](uint32_t bar) { return (CG == 2) ? mapa_shared(bar, 0) : bar; };
  // first output row of M-half h of tile t for this CTA, and the tile's first column
  // Tiles are visited in groups of group_m row tiles: inside a group the row
  // tile varies fastest, so the tiles in flight at any moment span a compact
  // block of rows x columns and share their A and B panels through L2.
  auto tile_coords = [&](int t, int& mb, int& n0) {
    const int gsz = args.group_m * n_tiles;
    const int first = (t / gsz) * args.group_m;
    const int gm = min(m_tiles - first, args.group_m);
    const int r = t - (first / args.group_m) * gsz;
    mb = (first + r % gm) * bm_pair + static_cast<int>(rank) * C::BM;
    n0 = (r / gm) * bn_out;
  };
  auto half_row = [&](int mb, int h) { return mb + h * C::BM * CG; };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < 2; ++i) {
        tma_prefetch_desc(&maps.a[i]);
        tma_prefetch_desc(&maps.la[i]);
        tma_prefetch_desc(&maps.lb[i]);
        if constexpr (ST) {
          tma_prefetch_desc(&maps.b[i]);
        } else {
          tma_prefetch_desc(&maps.codes[i]);
          tma_prefetch_desc(&maps.absmax[i]);
        }
      }
      auto load = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar_local, int x, int y) {
        if constexpr (CG == 2) tma_load_2d_pair(dst, m, leader(bar_local), x, y);
        else tma_load_2d(dst, m, bar_local, x, y);
      };
      int lora_bytes = MH * args.lora * C::LA_BYTES;
      if (MODE == MODE_FWD || MODE == MODE_FWD_GLU) lora_bytes += C::LBOP;
      if (MODE == MODE_BWD) lora_bytes += args.lora * C::LBOP;
      int j = 0, tl = 0;
      for (int t = cluster; t < total_tiles && ok; t += clusters, ++tl) {
        int mb, n0;
        tile_coords(t, mb, n0);
        for (int kb = 0; kb < nk; ++kb, ++j) {
          const int seg = kb >= args.nkb0 ? 1 : 0;
          const int kl = kb - seg * args.nkb0;
          // A operand tiles (complete on the leader's full barrier)
          const int s = j % C::S;
          ok = mbar_wait(empty_bar(s), ((j / C::S) & 1) ^ 1, args.status);
          if (!ok) break;
          if (rank == 0) mbar_arrive_expect_tx(full_bar(s), (C::A_BYTES + (ST ? C::B_BYTES : 0)) * CG);
          for (int h = 0; h < MH; ++h)
            load(sbase + C::OFF_A + s * C::A_BYTES + h * C::A_TILE, &maps.a[seg], full_bar(s), kl * 64,
                 half_row(mb, h));
          if constexpr (ST) {
            // staged weight: the B tile in the layout the dequantisers would write
            const uint32_t bdst = sbase + C::OFF_B + s * C::B_BYTES;
            if (MODE == MODE_BWD) {
              // W rows kl*64.. (the reduction index) x this CTA's BNC output columns, 64 per box
              for (int c = 0; c < C::BNC / 64; ++c)
                load(bdst + c * 8192, &maps.b[seg], full_bar(s), n0 + (int)rank * C::BNC + c * 64, kl * 64);
            } else {
              for (int bx = 0; bx < C::BNC / C::BOXR; ++bx) {
                const int p = (int)rank * C::BNC + bx * C::BOXR;  // first B row of the box in the pair tile
                int src = 0, row = n0 + p;
                if (MODE == MODE_FWD_GLU) {
                  src = p < C::BNT / 2 ? 0 : 1;
                  row = n0 + (src ? p - C::BNT / 2 : p);
                }
                load(bdst + bx * C::BOXR * 128, &maps.b[src], full_bar(s), kl * 64, row);
              }
            }
          }
        }
        if (!ok || args.lora == 0) continue;
        if constexpr (ST) {
          // LoRA operands as extra reduction blocks through the operand ring:
          // A slot <- s*XA (or s*G) [128 rows x 64], B slot <- the LoRA right factor;
          // ranks below 64 leave the rest of the boxes to the TMA's zero fill.
          // plain forward of fused projections: the tile's columns belong to one of them
          const int fop = (args.ncut[1] > 0 && n0 >= args.ncut[1]) ? 2 : ((args.ncut[0] > 0 && n0 >= args.ncut[0]) ? 1 : 0);
          const int fcol0 = fop == 0 ? 0 : (fop == 1 ? args.ncut[0] : args.ncut[1]);
          for (int i = 0; i < args.lora; ++i, ++j) {
            const int s = j % C::S;
            const int op = MODE == MODE_FWD ? fop : i;
            ok = mbar_wait(empty_bar(s), ((j / C::S) & 1) ^ 1, args.status);
            if (!ok) break;
            if (rank == 0) mbar_arrive_expect_tx(full_bar(s), (C::A_BYTES + C::B_BYTES) * CG);
            load(sbase + C::OFF_A + s * C::A_BYTES, &maps.la[op], full_bar(s), 0, half_row(mb, 0));
            const uint32_t bdst = sbase + C::OFF_B + s * C::B_BYTES;
            if (MODE == MODE_BWD) {
              // A_lora rows (this CTA's output columns) x rank, K-major
              for (int bx = 0; bx < C::BNC / C::BOXR; ++bx)
                load(bdst + bx * C::BOXR * 128, &maps.lb[op], full_bar(s), 0, n0 + (int)rank * C::BNC + bx * C::BOXR);
            } else {
              // B_lora [rank x columns], MN-major 64-column chunks; in the gated forward a chunk of
              // the other half is read from past the factor's last row, i.e. as zeros
              for (int c = 0; c < C::BNC / 64; ++c) {
                const int p = (int)rank * C::BNC + c * 64;
                int col = n0 + p - fcol0, y = 0;
                if (MODE == MODE_FWD_GLU) {
                  const int half = p < C::BNT / 2 ? 0 : 1;
                  col = n0 + (half ? p - C::BNT / 2 : p);
                  y = half == i ? 0 : 64;
                }
                load(bdst + c * 8192, &maps.lb[op], full_bar(s), col, y);
              }
            }
          }
          continue;
        }
        // LoRA operands of this tile (single buffer, released by the MMA's commit)
        ok = mbar_wait(lora_empty, (tl & 1) ^ 1, args.status);
        if (!ok) break;
        if (rank == 0) mbar_arrive_expect_tx(lora_full, lora_bytes * CG);
        for (int h = 0; h < MH; ++h)
          for (int i = 0; i < args.lora; ++i)
            load(sbase + C::OFF_LA + (h * 2 + i) * C::LA_BYTES, &maps.la[i], lora_full, 0, half_row(mb, h));
        if (MODE == MODE_FWD) {
          for (int c = 0; c < C::BNC / 64; ++c)
            load(sbase + C::OFF_LB + c * 2048, &maps.lb[0], lora_full, n0 + (int)rank * C::BNC + c * 64, 0);
        } else if (MODE == MODE_FWD_GLU) {
          for (int c = 0; c < C::BNC / 64; ++c) {
            const int p = (int)rank * C::BNC + c * 64;
            const int op = glu_chunk_is_gate(c) ? 0 : 1;
            load(sbase + C::OFF_LB + op * C::LBOP + c * 2048, &maps.lb[op], lora_full,
                 n0 + (op ? p - C::BNT / 2 : p), 0);
          }
        } else {
          for (int i = 0; i < args.lora; ++i)
            for (int bx = 0; bx < C::BNC / C::BOXR; ++bx)
              load(sbase + C::OFF_LB + i * C::LBOP + bx * C::BOXR * 32, &maps.lb[i], lora_full, 0,
                   n0 + (int)rank * C::BNC + bx * C::BOXR);
        }
      }
      if (!ok) settle_inflight();  // loads already issued land before the CTA can exit
    }
  } else if (warp == 2) {
    // ------------------------------------------------ raw-code producer --
    if constexpr (!ST) if (lane == 0) {
      bool ok = true;
      int j = 0;
      for (int t = cluster; t < total_tiles && ok; t += clusters) {
        int mb, n0;
        tile_coords(t, mb, n0);
        for (int kb = 0; kb < nk; ++kb, ++j) {
          const int seg = kb >= args.nkb0 ? 1 : 0;
          const int kl = kb - seg * args.nkb0;
          const int rs = j % C::RS;
          ok = mbar_wait(rempty_bar(rs), ((j / C::RS) & 1) ^ 1, args.status);
          if (!ok) break;
          mbar_arrive_expect_tx(rfull_bar(rs), C::RC_BYTES + C::RA_BYTES);
          const uint32_t rc = sbase + C::OFF_RC + rs * C::RC_BYTES;
          const uint32_t ra = sbase + C::OFF_RA + rs * C::RA_BYTES;
          if (MODE == MODE_BWD) {
            const int kw0 = n0 + (int)rank * C::BNC;
            tma_load_2d(rc, &maps.codes[seg], rfull_bar(rs), kw0 / 2, kl * 64);
            tma_load_2d(ra, &maps.absmax[seg], rfull_bar(rs), (kw0 / 64) & ~3, kl * 64);
          } else {
            for (int bx = 0; bx < C::BNC / C::BOXR; ++bx) {
              const int p = (int)rank * C::BNC + bx * C::BOXR;  // first B row of the box in the pair tile
              int src = 0, row = n0 + p;
              if (MODE == MODE_FWD_GLU) {
                src = p < C::BNT / 2 ? 0 : 1;
                row = n0 + (src ? p - C::BNT / 2 : p);
              }
              tma_load_2d(rc + bx * C::BOXR * 32, &maps.codes[src], rfull_bar(rs), kl * 32, row);
              tma_load_2d(ra + bx * C::BOXR * 16, &maps.absmax[src], rfull_bar(rs), kl & ~3, row);
            }
          }
        }
      }
      if (!ok) settle_inflight();
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA -----
    if (rank == 0 && lane == 0) {
      bool ok = true;
      const uint32_t idesc = idesc_bf16(C::BM * CG, C::BNT, false, MODE == MODE_BWD);
      const uint32_t idesc_lora = idesc_bf16(C::BM * CG, C::BNT, false, MODE != MODE_BWD);
      int j = 0, tl = 0;
      for (int t = cluster; t < total_tiles && ok; t += clusters, ++tl) {
        const int b = tl & 1;
        ok = mbar_wait(acc_empty0 + 8u * b, ((tl >> 1) & 1) ^ 1, args.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * 256;
        for (int kb = 0; kb < nk; ++kb, ++j) {
          const int s = j % C::S;
          ok = mbar_wait(full_bar(s), (j / C::S) & 1, args.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = sbase + C::OFF_A + s * C::A_BYTES;
          const uint32_t bs = sbase + C::OFF_B + s * C::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = (MODE == MODE_BWD) ? smem_desc(bs + kk * 2048, 8192, 1024, QL_SWZ_128B)
                                                   : smem_desc(bs + kk * 32, 16, 1024, QL_SWZ_128B);
#pragma unroll
            for (int h = 0; h < MH; ++h) {
              const uint64_t ad = smem_desc(a + h * C::A_TILE + kk * 32, 16, 1024, QL_SWZ_128B);
              umma_bf16<CG>(acc + h * C::BNT, ad, bd, idesc, (kb | kk) != 0);
            }
          }
          umma_commit<CG>(empty_bar(s));
        }
        if (!ok) break;
        if (ST && args.lora > 0) {
          for (int i = 0; i < args.lora && ok; ++i, ++j) {
            const int s = j % C::S;
            ok = mbar_wait(full_bar(s), (j / C::S) & 1, args.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a = sbase + C::OFF_A + s * C::A_BYTES;
            const uint32_t bs = sbase + C::OFF_B + s * C::B_BYTES;
            for (int kk = 0; kk < args.lora_k16; ++kk) {
              const uint64_t ad = smem_desc(a + kk * 32, 16, 1024, QL_SWZ_128B);
              const uint64_t bd = (MODE == MODE_BWD) ? smem_desc(bs + kk * 32, 16, 1024, QL_SWZ_128B)
                                                     : smem_desc(bs + kk * 2048, 8192, 1024, QL_SWZ_128B);
              umma_bf16<CG>(acc, ad, bd, idesc_lora, 1);
            }
            umma_commit<CG>(empty_bar(s));
          }
          if (!ok) break;
        } else if (args.lora > 0) {
          ok = mbar_wait(lora_full, tl & 1, args.status);
          if (!ok) break;
          tc_fence_after();
          for (int h = 0; h < MH; ++h) {
            for (int i = 0; i < args.lora; ++i) {
              const uint64_t ad = smem_desc(sbase + C::OFF_LA + (h * 2 + i) * C::LA_BYTES, 16, 256, QL_SWZ_32B);
              const uint64_t bd = (MODE == MODE_BWD)
                                      ? smem_desc(sbase + C::OFF_LB + i * C::LBOP, 16, 256, QL_SWZ_32B)
                                      : smem_desc(sbase + C::OFF_LB + i * C::LBOP, 2048, 1024, QL_SWZ_128B);
              umma_bf16<CG>(acc + h * C::BNT, ad, bd, idesc_lora, 1);
            }
          }
          umma_commit<CG>(lora_empty);
        }
        umma_commit<CG>(acc_full0 + 8u * b);
      }
      // let every issued MMA finish before TMEM can be released (after an error too)
      umma_commit<CG>(drain_bar);
      mbar_drain(drain_bar, 0);
    }
  } else if (warp < C::DQ_WARP0) {
    // ------------------------------------------------------ epilogue -----
    const int ew = warp - C::EPI_WARP0;  // 0..7
    const int lg = warp & 3;            // TMEM lane quadrant this warp may access
    const int half = ew >> 2;           // which half of the tile's column chunks
    const int row = lg * 32 + lane;
    // Staged gated backward: the saved e, g of this warp's next 32 x 32 chunk
    // are requested one chunk ahead (across tile boundaries too), so their
    // latency hides behind the current chunk and the wait for the next
    // accumulator.
    uint4 ec[4], gc[4];
    auto fetch_eg = [&](int t_, int it_) {
      int mb_, n0_;
      tile_coords(t_, mb_, n0_);
      constexpr int CPH = C::BNT / 32;
      const int grow_ = half_row(mb_, it_ / CPH) + row;
      const bool row_ok = grow_ < args.M;
      const size_t rbase = static_cast<size_t>(row_ok ? grow_ : 0) * args.ldo;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = n0_ + (it_ % CPH) * 32 + q * 8;
        const bool in = row_ok && col < args.N;
        ec[q] = in ? __ldg(reinterpret_cast<const uint4*>(args.Ein + rbase + col)) : make_uint4(0, 0, 0, 0);
        gc[q] = in ? __ldg(reinterpret_cast<const uint4*>(args.Gin + rbase + col)) : make_uint4(0, 0, 0, 0);
      }
    };
    if (ST && EPI == EPI_GLU_BWD && cluster < total_tiles) fetch_eg(cluster, half * 4);
    int tl = 0;
    for (int t = cluster; t < total_tiles; t += clusters, ++tl) {
      int mb, n0;
      tile_coords(t, mb, n0);
      const int b = tl & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full0 + 8u * b, (tl >> 1) & 1, args.status))) break;
      tc_fence_after();
      const uint32_t tacc = tmem + b * 256 + (static_cast<uint32_t>(lg * 32) << 16);
      if constexpr (ST) {
        // Output chunks (32 rows x 32 columns) go through this warp's shared
        // slots and leave by TMA store, which writes whole lines and clips at
        // the tensor's edges.
        const uint32_t stg = sbase + C::OFF_EPI + ew * 3 * C::EPI_SLOT;
        const uint64_t pol = l2_policy_evict_first();
        uint8_t* stg_g = sgen + C::OFF_EPI + ew * 3 * C::EPI_SLOT;
        // byte offset of 16-byte chunk q of this lane's row (64B swizzle)
        auto soff = [&](int q) { return lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4); };
        auto put = [&](int slot, int q, uint4 v) {
          *reinterpret_cast<uint4*>(stg_g + slot * C::EPI_SLOT + soff(q)) = v;
        };
        if (EPI == EPI_STORE || EPI == EPI_GLU_BWD) {
          constexpr int CPH = C::BNT / 32;  // 32-column chunks per M-half
#pragma unroll 1
          for (int it = half * 4; it < half * 4 + 4; ++it) {
            const int h = it / CPH, c = it % CPH;
            const int grow0 = half_row(mb, h) + lg * 32;
            const int col0 = n0 + c * 32;
            uint4 ecur[4], gcur[4];
            if (EPI == EPI_GLU_BWD) {
#pragma unroll
              for (int q = 0; q < 4; ++q) ecur[q] = ec[q], gcur[q] = gc[q];
              if (it + 1 < half * 4 + 4) fetch_eg(t, it + 1);
              else if (t + clusters < total_tiles) fetch_eg(t + clusters, half * 4);
            }
            float v[32];
            tmem_ld_32x32b_x32(tacc + h * C::BNT + c * 32, v);
            if (lane == 0) bulk_wait_group_read<0>();  // the previous chunk's stores have read the slots
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (EPI == EPI_STORE) {
                uint4 o;
                o.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
                o.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
                o.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
                o.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
                put(0, q, o);
              } else {
                const uint32_t ewv[4] = {ecur[q].x, ecur[q].y, ecur[q].z, ecur[q].w};
                const uint32_t gwv[4] = {gcur[q].x, gcur[q].y, gcur[q].z, gcur[q].w};
                uint32_t de[4], dg[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float f0, d0, f1, d1;
                  const float e0 = bf16_lo(ewv[i]), e1 = bf16_hi(ewv[i]);
                  const float g0 = bf16_lo(gwv[i]), g1 = bf16_hi(gwv[i]);
                  act_fg(args.act, e0, f0, d0);
                  act_fg(args.act, e1, f1, d1);
                  const float h0 = v[q * 8 + 2 * i], h1 = v[q * 8 + 2 * i + 1];
                  de[i] = pack_bf16x2(h0 * g0 * d0, h1 * g1 * d1);
                  dg[i] = pack_bf16x2(h0 * f0, h1 * f1);
                }
                put(0, q, make_uint4(de[0], de[1], de[2], de[3]));
                put(1, q, make_uint4(dg[0], dg[1], dg[2], dg[3]));
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out[0], stg, col0, grow0, pol);
              if (EPI == EPI_GLU_BWD) tma_store_2d(&maps.out[1], stg + C::EPI_SLOT, col0, grow0, pol);
              bulk_commit_group();
            }
          }
        } else {  // EPI_GLU_FWD: per M-half, columns [0, BNT/2) hold e and [BNT/2, BNT) hold g
          constexpr int CPH = C::BNT / 64;
#pragma unroll 1
          for (int it = half * 2; it < half * 2 + 2; ++it) {
            const int h = it / CPH, c = it % CPH;
            const int grow0 = half_row(mb, h) + lg * 32;
            const int col0 = n0 + c * 32;
            float e[32], g[32];
            tmem_ld_32x32b_x32(tacc + h * C::BNT + c * 32, e);
            tmem_ld_32x32b_x32(tacc + h * C::BNT + C::BNT / 2 + c * 32, g);
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t ewv[4], gwv[4], hwv[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float e0 = e[q * 8 + 2 * i], e1 = e[q * 8 + 2 * i + 1];
                const float g0 = g[q * 8 + 2 * i], g1 = g[q * 8 + 2 * i + 1];
                ewv[i] = pack_bf16x2(e0, e1);
                gwv[i] = pack_bf16x2(g0, g1);
                hwv[i] = pack_bf16x2(act_f(args.act, e0) * g0, act_f(args.act, e1) * g1);
              }
              put(0, q, make_uint4(ewv[0], ewv[1], ewv[2], ewv[3]));
              put(1, q, make_uint4(gwv[0], gwv[1], gwv[2], gwv[3]));
              put(2, q, make_uint4(hwv[0], hwv[1], hwv[2], hwv[3]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out[0], stg, col0, grow0, pol);
              tma_store_2d(&maps.out[1], stg + C::EPI_SLOT, col0, grow0, pol);
              tma_store_2d(&maps.out[2], stg + 2 * C::EPI_SLOT, col0, grow0, pol);
              bulk_commit_group();
            }
          }
        }
      } else {
        if (EPI == EPI_STORE || EPI == EPI_GLU_BWD) {
          constexpr int CPH = C::BNT / 32;  // 32-column chunks per M-half
  #pragma unroll 1
          for (int it = half * 4; it < half * 4 + 4; ++it) {
            const int h = it / CPH, c = it % CPH;
            const int grow = half_row(mb, h) + row;
            const bool row_ok = grow < args.M;
            const size_t rbase = static_cast<size_t>(row_ok ? grow : 0) * args.ldo;
            uint4 ec[4], gc[4];
            if (EPI == EPI_GLU_BWD) {
              // the chunk's saved e, g are requested before its TMEM load so the two latencies overlap
  #pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = n0 + c * 32 + q * 8;
                const bool in = row_ok && col < args.N;
                ec[q] = in ? __ldg(reinterpret_cast<const uint4*>(args.Ein + rbase + col)) : make_uint4(0, 0, 0, 0);
                gc[q] = in ? __ldg(reinterpret_cast<const uint4*>(args.Gin + rbase + col)) : make_uint4(0, 0, 0, 0);
              }
            }
            float v[32];
            tmem_ld_32x32b_x32(tacc + h * C::BNT + c * 32, v);
            if (!row_ok) continue;
  #pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = n0 + c * 32 + q * 8;
              if (col >= args.N) break;
              if (EPI == EPI_STORE) {
                uint4 o;
                o.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
                o.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
                o.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
                o.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
                *reinterpret_cast<uint4*>(args.D + rbase + col) = o;
              } else {
                const uint32_t ewv[4] = {ec[q].x, ec[q].y, ec[q].z, ec[q].w};
                const uint32_t gwv[4] = {gc[q].x, gc[q].y, gc[q].z, gc[q].w};
                uint32_t de[4], dg[4];
  #pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float f0, d0, f1, d1;
                  const float e0 = bf16_lo(ewv[i]), e1 = bf16_hi(ewv[i]);
                  const float g0 = bf16_lo(gwv[i]), g1 = bf16_hi(gwv[i]);
                  act_fg(args.act, e0, f0, d0);
                  act_fg(args.act, e1, f1, d1);
                  const float h0 = v[q * 8 + 2 * i], h1 = v[q * 8 + 2 * i + 1];
                  de[i] = pack_bf16x2(h0 * g0 * d0, h1 * g1 * d1);
                  dg[i] = pack_bf16x2(h0 * f0, h1 * f1);
                }
                *reinterpret_cast<uint4*>(args.dE + rbase + col) = make_uint4(de[0], de[1], de[2], de[3]);
                *reinterpret_cast<uint4*>(args.dG + rbase + col) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
              }
            }
          }
        } else {  // EPI_GLU_FWD: per M-half, columns [0, BNT/2) hold e and [BNT/2, BNT) hold g
          constexpr int CPH = C::BNT / 64;  // (e, g) chunk pairs per M-half
  #pragma unroll 1
          for (int it = half * 2; it < half * 2 + 2; ++it) {
            const int h = it / CPH, c = it % CPH;
            const int grow = half_row(mb, h) + row;
            const bool row_ok = grow < args.M;
            const size_t rbase = static_cast<size_t>(row_ok ? grow : 0) * args.ldo;
            float e[32], g[32];
            tmem_ld_32x32b_x32(tacc + h * C::BNT + c * 32, e);
            tmem_ld_32x32b_x32(tacc + h * C::BNT + C::BNT / 2 + c * 32, g);
            if (!row_ok) continue;
  #pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = n0 + c * 32 + q * 8;
              if (col >= args.N) break;
              uint32_t ewv[4], gwv[4], hwv[4];
  #pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float e0 = e[q * 8 + 2 * i], e1 = e[q * 8 + 2 * i + 1];
                const float g0 = g[q * 8 + 2 * i], g1 = g[q * 8 + 2 * i + 1];
                ewv[i] = pack_bf16x2(e0, e1);
                gwv[i] = pack_bf16x2(g0, g1);
                hwv[i] = pack_bf16x2(act_f(args.act, e0) * g0, act_f(args.act, e1) * g1);
              }
              *reinterpret_cast<uint4*>(args.E + rbase + col) = make_uint4(ewv[0], ewv[1], ewv[2], ewv[3]);
              *reinterpret_cast<uint4*>(args.G + rbase + col) = make_uint4(gwv[0], gwv[1], gwv[2], gwv[3]);
              *reinterpret_cast<uint4*>(args.H + rbase + col) = make_uint4(hwv[0], hwv[1], hwv[2], hwv[3]);
            }
          }
        }
      }
      // accumulator b may be overwritten once every epilogue warp of the pair is done with it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2) mbar_arrive_cluster(leader(acc_empty0 + 8u * b));
        else mbar_arrive(acc_empty0 + 8u * b);
      }
    }
    if (ST && lane == 0) bulk_wait_group<0>();  // output stores complete before the CTA exits
  } else if constexpr (!ST) {
    // --------------------------------------------------- dequantisers ----
    const int dq = (warp - C::DQ_WARP0) * 32 + lane;  // 0..255
    constexpr int groups = 256 / C::NB;
    const int grp = dq / C::NB;
    const int tq = dq % C::NB;
    int j = 0;
    bool ok = true;
    for (int t = cluster; t < total_tiles && ok; t += clusters) {
      int mb, n0;
      tile_coords(t, mb, n0);
      for (int kb = 0; kb < nk; ++kb, ++j) {
        if (j % groups != grp) continue;
        const int seg = kb >= args.nkb0 ? 1 : 0;
        const int kl = kb - seg * args.nkb0;
        const int rs = j % C::RS;
        ok = __all_sync(0xffffffffu, mbar_wait(rfull_bar(rs), (j / C::RS) & 1, args.status));
        if (!ok) break;
        const uint8_t* rc = sgen + C::OFF_RC + rs * C::RC_BYTES;
        const float* ra = reinterpret_cast<const float*>(sgen + C::OFF_RA + rs * C::RA_BYTES);
        uint4 w0, w1;
        float amax;
        int r = 0, cchunk = 0;
        if (MODE == MODE_BWD) {
          // raw tile: 64 rows x (BNC/2) bytes with the matching TMA swizzle (128B, 64B or 32B)
          r = tq & 63;
          cchunk = tq >> 6;
          constexpr int RB = C::BNC / 2;
          constexpr int SHIFT = (RB == 128) ? 0 : (RB == 64 ? 1 : 2);
          constexpr int MASK = RB / 16 - 1;
          const int x = (r >> SHIFT) & MASK;
          w0 = *reinterpret_cast<const uint4*>(rc + r * RB + (((2 * cchunk) ^ x) << 4));
          w1 = *reinterpret_cast<const uint4*>(rc + r * RB + (((2 * cchunk + 1) ^ x) << 4));
          amax = ra[r * 4 + (((n0 + (int)rank * C::BNC) / 64) & 3) + cchunk];
        } else {
          // raw tile: NB rows x 32 bytes, 32B swizzle
          r = tq;
          const int x = (r >> 2) & 1;
          w0 = *reinterpret_cast<const uint4*>(rc + r * 32 + ((0 ^ x) << 4));
          w1 = *reinterpret_cast<const uint4*>(rc + r * 32 + ((1 ^ x) << 4));
          amax = ra[r * 4 + (kl & 3)];
        }
        const int s = j % C::S;
        ok = __all_sync(0xffffffffu, mbar_wait(empty_bar(s), ((j / C::S) & 1) ^ 1, args.status));
        if (!ok) break;
        uint32_t tlo[4], thi[4];
        nf4_block_table(amax, tlo, thi);
        uint8_t* bt = sgen + C::OFF_B + s * C::B_BYTES;
        uint8_t* dst = (MODE == MODE_BWD) ? bt + cchunk * 8192 + (r >> 3) * 1024 + (r & 7) * 128
                                          : bt + (r >> 3) * 1024 + (r & 7) * 128;
        const int x7 = r & 7;
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(dst + ((i ^ x7) << 4)) = nf4_decode8(wv[i], tlo, thi);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 2) mbar_arrive_cluster(leader(full_bar(s)));
          else mbar_arrive(full_bar(s));
          // The raw slot is released only now: the stores above consumed every
          // value loaded from it, so those shared-memory loads have returned
          // before the TMA may overwrite the slot (an mbarrier arrive issued
          // right after the loads could overtake them).
          mbar_arrive(rempty_bar(rs));
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown --
  __syncwarp();  // lanes that skipped a role's single-thread loop wait for it here
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<CG>(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- launch --
template <int MODE, int EPI, int CG, int MH, bool ST>
static cudaError_t launch_one(const GemmMaps& maps, const GemmArgs& args, cudaStream_t stream) {
  using C = GemmCfg<MODE, CG, MH, ST>;
  auto kern = gemm_nf4_kernel<MODE, EPI, CG, MH, ST>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int resident[64] = {0};  // co-resident CTAs (multiple of CG) per device, per instantiation
  const int bn_out = (EPI == EPI_GLU_FWD) ? C::BNT / 2 : C::BNT;
  const int bm_pair = C::BM * CG * MH;
  const int n_tiles = (args.N + bn_out - 1) / bn_out;
  const int m_tiles = (args.M + bm_pair - 1) / bm_pair;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!resident[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int n = sms / CG;
    if (CG > 1) {
      cfg.gridDim = dim3(static_cast<unsigned>(sms - sms % CG), 1, 1);
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0 && clusters < n)
        n = clusters;
      cudaGetLastError();
    }
    resident[dev] = n * CG;
  }
  const int total = m_tiles * n_tiles;
  const int ctas = apply_grid_cap((total * CG < resident[dev]) ? total * CG : resident[dev], CG);
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, maps, args);
}

// Tile configurations: 1 = single CTA 128 x 256, 2 = CTA pair 256 x 256,
// 3 = CTA pair 512 x 128 (all three dequantising in the mainloop);
// 4 = CTA pair 256 x 256 fed from a staged bf16 weight (maps.b).
cudaError_t launch_gemm_nf4(int mode, int epi, int tiles, const GemmMaps& maps, const GemmArgs& args,
                            cudaStream_t stream) {
#define QL_CASE(M_, E_)                                                          \
  if (mode == M_ && epi == E_) {                                                 \
    if (tiles == 1) return launch_one<M_, E_, 1, 1, false>(maps, args, stream);  \
    if (tiles == 2) return launch_one<M_, E_, 2, 1, false>(maps, args, stream);  \
    if (tiles == 3) return launch_one<M_, E_, 2, 2, false>(maps, args, stream);  \
    if (tiles == 4) return launch_one<M_, E_, 2, 1, true>(maps, args, stream);   \
  }
  QL_CASE(MODE_FWD, EPI_STORE)
  QL_CASE(MODE_FWD_GLU, EPI_GLU_FWD)
  QL_CASE(MODE_BWD, EPI_STORE)
  QL_CASE(MODE_BWD, EPI_GLU_BWD)
#undef QL_CASE
  return cudaErrorInvalidValue;
}

// Columns of B each CTA dequantises for a tile configuration (host-side tensor map boxes).
int gemm_nf4_b_cols_per_cta(int tiles) { return tiles == 1 ? 256 : (tiles == 3 ? 64 : 128); }

}  // namespace ql
