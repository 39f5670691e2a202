// ffn_sm100.cuh -- blockwise feedforward, bf16, sm_100a.
//
// A host of the ring "computes attention and feedforward for its query
// block block by block", and the blockwise feedforward is what lowers the
// feedforward's share of activation memory (Ring Attention with Blockwise
// Transformers for Near-Infinite Context, Summary and Key points).  The
// feedforward here is Llama's gated SiLU unit:
//   H   = silu(X W_gate^T) * (X W_up^T)        [rows, f]
//   out = H W_down^T                           [rows, h]
// computed one block of token rows at a time (the host loops over blocks),
// so [rows, f] intermediates exist for one block only.  Backward of
// sum(dout * out), per block, with G/U recomputed from X:
//   dH = dout W_down;  dU = dH * silu(G);  dG = dH * U * silu'(G)
//   dX = dG W_gate + dU W_up
//   dW_gate += dG^T X;  dW_up += dU^T X;  dW_down += dout^T H
//
// Every product is C = A B^T (A: M x K, B: N x K), on one persistent kernel:
//   * CTA tile 128 x 256 output, K steps of 64, a 4-stage TMA ring (A 16 KB
//     + B 32 KB per stage).  An operand is K-major (its rows run along K:
//     boxes of 64 K x 128 rows) or MN-major (stored K rows by M or N
//     columns, e.g. dG^T: boxes of 64 columns x 64 K rows, 8 KB atoms);
//   * warp 0: TMA producer; warp 1: TMEM owner, lane 0 issues the
//     tcgen05.mma (M = 128, N = 256, four K = 16 steps per stage); warps
//     2-5: epilogue, one output row per thread (its TMEM lane);
//   * two 256-column fp32 accumulators in TMEM (all 512 columns), so the
//     epilogue of one tile runs while the next tile's products accumulate;
//   * tiles are visited in bands of group_m row tiles, column by column, so
//     the tiles in flight share their A rows and B columns in L2 (the host
//     picks the band per product: a whole block of rows when the weights are
//     the large operand, so each weight column is read once per block; one
//     row tile when B is small enough to stay in L2 whole).
// Epilogues: EPI_STORE -- 256 columns as bf16; EPI_SWIGLU -- the B stage
// holds 128 rows of W_gate then 128 rows of W_up for the same columns and
// the epilogue writes silu(gate) * up (128 columns); EPI_SWIGLU_BWD -- the
// same product, and the epilogue reads dH and writes dG, dU and H (zeros
// for rows past M, so later products over whole 64-row K steps add
// nothing from them); EPI_ACC32 -- adds the 256 columns into a float32
// output (two stacked outputs split at row m_split: dW_gate and dW_up come
// from one product over [dG | dU]).  Split K: the first half of K comes from (A0, B0), the second
// from (A1, B1).  Rows past M are computed from zero-filled rows and not
// stored.
#pragma once

#include "ptx.cuh"

namespace lca {

namespace ffn {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kGroupM = 16;  // default band height (row tiles)
constexpr int kThreads = 192;
constexpr uint32_t kAStage = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBHalf = 128 * kBK * 2;   // 16 KB
constexpr uint32_t kBStage = 2 * kBHalf;     // 32 KB
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kAStage;
constexpr uint32_t kOffBar = kOffB + kStages * kBStage;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack

enum { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_SWIGLU_BWD = 2, EPI_ACC32 = 3 };

enum {
  B_FULL = 0,                 // + stage
  B_EMPTY = B_FULL + kStages, // + stage
  B_ACCFULL = B_EMPTY + kStages,   // + accumulator
  B_ACCEMPTY = B_ACCFULL + 2,      // + accumulator, 128 arrivals
  B_DRAIN = B_ACCEMPTY + 2,
  NUM_BARS
};

struct Args {
  int M;             // rows of C (rows past M are not stored)
  int K;             // reduction length, a multiple of 64 (of 128 when split)
  int n_tm, n_tn;    // tiles along M and N
  int a_off;         // A coordinate offset: rows (K-major) or K rows (MN-major)
  int b_off;         // B coordinate offset, likewise
  int ldo;           // row stride of the outputs, in elements
  int ldo3;          // row stride of out3
  int ld_in;         // row stride of `in`
  int m_split;       // EPI_ACC32: rows from m_split on go to out32b (ignored when
                     // out32b is null)
  int group_m;       // band height of the tile raster in row tiles (>= 1)
  unsigned long long budget;
  __nv_bfloat16* out;   // C (EPI_STORE, EPI_SWIGLU), dG (EPI_SWIGLU_BWD)
  __nv_bfloat16* out2;  // dU (EPI_SWIGLU_BWD)
  __nv_bfloat16* out3;  // H (EPI_SWIGLU_BWD)
  const __nv_bfloat16* in;  // dH (EPI_SWIGLU_BWD)
  float* out32;         // EPI_ACC32: C += A B^T (rows below m_split)
  float* out32b;        // EPI_ACC32: rows from m_split on, counted from m_split
};

// Tile t -> (tm, tn): bands of group_m row tiles, column by column.
__host__ __device__ inline void tile_coords(int t, int n_tm, int n_tn, int group_m, int& tm,
                                            int& tn) {
  const int band = t / (group_m * n_tn);
  const int first = band * group_m;
  const int gm = n_tm - first < group_m ? n_tm - first : group_m;
  const int t_in = t - band * group_m * n_tn;
  tm = first + t_in % gm;
  tn = t_in / gm;
}

}  // namespace ffn

// One 128 x 256 tile's epilogue rows for the four epilogues (one output
// row per thread; every lane takes part in the TMEM loads).
template <int kEpi>
__device__ __forceinline__ void ffn_epilogue(const ffn::Args& a, uint32_t acc, int row, int tn) {
  using namespace ffn;
  const bool row_in = row < a.M;
  const float kLog2e = 1.4426950408889634f;
  const size_t orow = static_cast<size_t>(row_in ? row : 0) * a.ldo;
  if constexpr (kEpi == EPI_STORE) {
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      __syncwarp();
      tmem_ld32(acc + c * 32, v);
      if (row_in) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + orow + tn * kBN + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]),
                              pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                              pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                              pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      }
    }
  } else if constexpr (kEpi == EPI_SWIGLU) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float g[32], u[32];
      __syncwarp();
      tmem_ld32(acc + c * 32, g);
      tmem_ld32(acc + 128 + c * 32, u);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float s0 = g[2 * i] * __frcp_rn(1.f + ex2_approx(-g[2 * i] * kLog2e));
        const float s1 = g[2 * i + 1] * __frcp_rn(1.f + ex2_approx(-g[2 * i + 1] * kLog2e));
        pk[i] = pack_bf16x2(s0 * u[2 * i], s1 * u[2 * i + 1]);
      }
      if (row_in) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + orow + tn * 128 + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    }
  } else if constexpr (kEpi == EPI_SWIGLU_BWD) {
    // rows past M (inside the block's last tile) are written as zeros
    const size_t wrow = static_cast<size_t>(row) * a.ldo;
    const size_t hrow = static_cast<size_t>(row) * a.ldo3;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float g[32], u[32];
      __syncwarp();
      tmem_ld32(acc + c * 32, g);
      tmem_ld32(acc + 128 + c * 32, u);
      const int col = tn * 128 + c * 32;
      uint32_t dh[16];
      if (row_in) {
        const uint4* src =
            reinterpret_cast<const uint4*>(a.in + static_cast<size_t>(row) * a.ld_in + col);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = src[q];
          dh[4 * q] = w.x;
          dh[4 * q + 1] = w.y;
          dh[4 * q + 2] = w.z;
          dh[4 * q + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) dh[i] = 0u;
      }
      uint32_t pg[16], pu[16], ph[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float gv[2], dd[2], rg[2], ru[2], rh[2];
        gv[0] = g[2 * i];
        gv[1] = g[2 * i + 1];
        dd[0] = __uint_as_float(dh[i] << 16);
        dd[1] = __uint_as_float(dh[i] & 0xffff0000u);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float sg = __frcp_rn(1.f + ex2_approx(-gv[e] * kLog2e));  // sigmoid
          const float sl = gv[e] * sg;                                     // silu
          const float uv = u[2 * i + e];
          ru[e] = dd[e] * sl;
          rg[e] = dd[e] * uv * sg * (1.f + gv[e] * (1.f - sg));
          rh[e] = row_in ? sl * uv : 0.f;
        }
        pg[i] = pack_bf16x2(rg[0], rg[1]);
        pu[i] = pack_bf16x2(ru[0], ru[1]);
        ph[i] = pack_bf16x2(rh[0], rh[1]);
      }
      uint4* dg = reinterpret_cast<uint4*>(a.out + wrow + col);
      uint4* du = reinterpret_cast<uint4*>(a.out2 + wrow + col);
      uint4* hh = reinterpret_cast<uint4*>(a.out3 + hrow + col);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        dg[q] = make_uint4(pg[4 * q], pg[4 * q + 1], pg[4 * q + 2], pg[4 * q + 3]);
        du[q] = make_uint4(pu[4 * q], pu[4 * q + 1], pu[4 * q + 2], pu[4 * q + 3]);
        hh[q] = make_uint4(ph[4 * q], ph[4 * q + 1], ph[4 * q + 2], ph[4 * q + 3]);
      }
    }
  } else {  // EPI_ACC32
    // two stacked outputs: a 128-row tile lies wholly on one side of m_split.
    // Without a second output (out32b null) every row goes to out32, whatever
    // m_split holds.
    float* base = (row < a.m_split || a.out32b == nullptr)
                      ? a.out32 + orow
                      : a.out32b + static_cast<size_t>(row - a.m_split) * a.ldo;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      __syncwarp();
      tmem_ld32(acc + c * 32, v);
      if (row_in) {
        float4* dst = reinterpret_cast<float4*>(base + tn * kBN + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 o = dst[q];
          o.x += v[4 * q];
          o.y += v[4 * q + 1];
          o.z += v[4 * q + 2];
          o.w += v[4 * q + 3];
          dst[q] = o;
        }
      }
    }
  }
}

// kAmn / kBmn: the operand is MN-major.  kSplit: K's first half from
// (A0, B0), its second half from (A1, B1).
template <int kEpi, bool kAmn, bool kBmn, bool kSplit>
__global__ void __launch_bounds__(ffn::kThreads, 1)
    ffn_gemm_sm100(const __grid_constant__ CUtensorMap tmA0,
                   const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ ffn::Args a) {
  using namespace ffn;
  constexpr bool kGateUp = kEpi == EPI_SWIGLU || kEpi == EPI_SWIGLU_BWD;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, kAmn, kBmn);
  // MN-major atoms: 64 columns x 64 K rows, 8 KB apart
  constexpr uint32_t kAtom = 64 * kBK * 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sA = base + kOffA, sB = base + kOffB;
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * NUM_BARS + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = a.n_tm * a.n_tn;
  const int nk = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i)
      mbar_init(bar(i), (i == B_ACCEMPTY || i == B_ACCEMPTY + 1) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtl wc{abort_flag, a.budget};

  if (warp == 0) {
    // =================================================== TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmB0);
      if (kSplit) tma_prefetch_desc(&tmA1);
      if (kSplit || kGateUp) tma_prefetch_desc(&tmB1);
      int issued[kStages] = {};
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, a.n_tm, a.n_tn, a.group_m, tm, tn);
        const int m0 = tm * kBM;
        // first B row/column of the tile: 256 output columns, or 128 gate +
        // 128 up rows for the same 128 columns
        const int n0 = kGateUp ? tn * 128 : tn * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages) ok = wait_bar(bar(B_EMPTY + s), ((it / kStages) - 1) & 1, wc, 601);
          if (!ok) break;
          const bool second = kSplit && kb >= nk / 2;
          const CUtensorMap* mA = second ? &tmA1 : &tmA0;
          const CUtensorMap* mB = second ? &tmB1 : &tmB0;
          const int k0 = (second ? kb - nk / 2 : kb) * kBK;
          const uint32_t fb = bar(B_FULL + s);
          const uint32_t as = sA + s * kAStage, bs = sB + s * kBStage;
          mbar_expect_tx(fb, kAStage + kBStage);
          if (kAmn) {
            tma_load_2d(as, mA, fb, m0, a.a_off + k0);
            tma_load_2d(as + kAtom, mA, fb, m0 + 64, a.a_off + k0);
          } else {
            tma_load_2d(as, mA, fb, k0, a.a_off + m0);
          }
          if (kBmn) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d(bs + j * kAtom, mB, fb, n0 + 64 * j, a.b_off + k0);
          } else if (kGateUp) {
            tma_load_2d(bs, &tmB0, fb, k0, a.b_off + n0);
            tma_load_2d(bs + kBHalf, &tmB1, fb, k0, a.b_off + n0);
          } else {
            tma_load_2d(bs, mB, fb, k0, a.b_off + n0);
            tma_load_2d(bs + kBHalf, mB, fb, k0, a.b_off + n0 + 128);
          }
          ++issued[s];
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) drain_bar(bar(B_FULL + s), (issued[s] - 1) & 1, 181);
      }
    }
  } else if (warp == 1) {
    // =================================================== MMA issuer
    if (lane == 0) {
      int it = 0, li = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++li) {
        const int b = li & 1;
        if (li >= 2) ok = wait_bar(bar(B_ACCEMPTY + b), ((li >> 1) - 1) & 1, wc, 611);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          ok = wait_bar(bar(B_FULL + s), (it / kStages) & 1, wc, 612);
          if (!ok) break;
          tc_fence_after();
          const uint32_t as = sA + s * kAStage, bs = sB + s * kBStage;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // K-major: 16 K elements = 32 bytes along each row; MN-major: 16
            // K rows = 2048 bytes, atoms kAtom apart
            const uint64_t ad = kAmn ? sdesc_sw128(as + kk * 2048, kAtom, 1024)
                                     : sdesc_sw128(as + kk * 32, 16, 1024);
            const uint64_t bd = kBmn ? sdesc_sw128(bs + kk * 2048, kAtom, 1024)
                                     : sdesc_sw128(bs + kk * 32, 16, 1024);
            mma_bf16_ss(acc, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_EMPTY + s));
        }
        if (!ok) break;
        tc_commit(bar(B_ACCFULL + b));
      }
      // wait for every product this thread issued before TMEM is freed
      tc_commit(bar(B_DRAIN));
      drain_bar(bar(B_DRAIN), 0, 182);
    }
  } else {
    // =================================================== epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const uint32_t lad = static_cast<uint32_t>(q * 32) << 16;
    int li = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++li) {
      const int b = li & 1;
      if (!__all_sync(0xffffffffu, wait_bar(bar(B_ACCFULL + b), (li >> 1) & 1, wc, 621))) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, a.n_tm, a.n_tn, a.group_m, tm, tn);
      ffn_epilogue<kEpi>(a, tmem + lad + b * kBN, tm * kBM + r, tn);
      // this accumulator may be overwritten by the tile after next
      tc_fence_before();
      mbar_arrive(bar(B_ACCEMPTY + b));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace lca
