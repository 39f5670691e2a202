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
// so the [rows, f] intermediate exists for one block only.
//
// Both products are C = A B^T with A [M, K] and B [N, K] row-major (every
// operand K-major), on one persistent kernel:
//   * CTA tile 128 x 256 output, K steps of 64 (one 128-byte swizzle atom),
//     a 4-stage TMA ring (A 16 KB + B 32 KB per stage);
//   * warp 0: TMA producer; warp 1: TMEM owner, lane 0 issues the
//     tcgen05.mma (M = 128, N = 256, four K = 16 steps per stage); warps
//     2-5: epilogue, one output row per thread (its TMEM lane);
//   * two 256-column fp32 accumulators in TMEM (all 512 columns), so the
//     epilogue of one tile runs while the next tile's products accumulate;
//   * tiles are visited in bands of 16 row tiles, column by column, so the
//     tiles in flight share their A rows and B columns in L2.
// Epilogues: EPI_SWIGLU -- the B stage holds 128 rows of W_gate then 128
// rows of W_up for the same output columns, and the epilogue writes
// silu(gate) * up as bf16 (128 columns per tile); EPI_STORE -- the 256
// columns as bf16.  Rows past M are computed from zero-filled A rows and
// not stored.
#pragma once

#include "ptx.cuh"

namespace lca {

namespace ffn {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kGroupM = 16;
constexpr int kThreads = 192;
constexpr uint32_t kAStage = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBHalf = 128 * kBK * 2;   // 16 KB
constexpr uint32_t kBStage = 2 * kBHalf;     // 32 KB
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kAStage;
constexpr uint32_t kOffBar = kOffB + kStages * kBStage;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack

enum { EPI_STORE = 0, EPI_SWIGLU = 1 };

enum {
  B_FULL = 0,                 // + stage
  B_EMPTY = B_FULL + kStages, // + stage
  B_ACCFULL = B_EMPTY + kStages,   // + accumulator
  B_ACCEMPTY = B_ACCFULL + 2,      // + accumulator, 128 arrivals
  B_DRAIN = B_ACCEMPTY + 2,
  NUM_BARS
};

constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, false, false);

struct Args {
  int M;             // rows of C (rows past M are not stored)
  int K;             // reduction length, a multiple of 64
  int n_tm, n_tn;    // tiles along M and N
  int a_row0;        // first A row (tensor-map coordinate) of this launch
  int ldo;           // row stride of out, in elements
  unsigned long long budget;
  __nv_bfloat16* out;  // C row 0, column 0
};

// Tile t -> (tm, tn): bands of kGroupM row tiles, column by column.
__device__ __forceinline__ void tile_coords(int t, int n_tm, int n_tn, int& tm, int& tn) {
  const int band = t / (kGroupM * n_tn);
  const int first = band * kGroupM;
  const int gm = n_tm - first < kGroupM ? n_tm - first : kGroupM;
  const int t_in = t - band * kGroupM * n_tn;
  tm = first + t_in % gm;
  tn = t_in / gm;
}

}  // namespace ffn

template <int kEpi>
__global__ void __launch_bounds__(ffn::kThreads, 1)
    ffn_gemm_sm100(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ ffn::Args a) {
  using namespace ffn;
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
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      if (kEpi == EPI_SWIGLU) tma_prefetch_desc(&tmB1);
      int issued[kStages] = {};
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, a.n_tm, a.n_tn, tm, tn);
        const int arow = a.a_row0 + tm * kBM;
        // B rows of this tile: 256 output columns, or 128 gate + 128 up rows
        const int brow0 = kEpi == EPI_SWIGLU ? tn * 128 : tn * kBN;
        const int brow1 = kEpi == EPI_SWIGLU ? tn * 128 : tn * kBN + 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages) ok = wait_bar(bar(B_EMPTY + s), ((it / kStages) - 1) & 1, wc, 601);
          if (!ok) break;
          const uint32_t fb = bar(B_FULL + s);
          mbar_expect_tx(fb, kAStage + kBStage);
          tma_load_2d(sA + s * kAStage, &tmA, fb, kb * kBK, arow);
          tma_load_2d(sB + s * kBStage, &tmB0, fb, kb * kBK, brow0);
          tma_load_2d(sB + s * kBStage + kBHalf, kEpi == EPI_SWIGLU ? &tmB1 : &tmB0, fb,
                      kb * kBK, brow1);
          ++issued[s];
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) drain_bar(bar(B_FULL + s), (issued[s] - 1) & 1, a.budget);
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
            mma_bf16_ss(acc, sdesc_sw128(as + kk * 32, 16, 1024),
                        sdesc_sw128(bs + kk * 32, 16, 1024), kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_EMPTY + s));
        }
        if (!ok) break;
        tc_commit(bar(B_ACCFULL + b));
      }
      // wait for every product this thread issued before TMEM is freed
      tc_commit(bar(B_DRAIN));
      drain_bar(bar(B_DRAIN), 0, a.budget);
    }
  } else {
    // =================================================== epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const uint32_t lad = static_cast<uint32_t>(q * 32) << 16;
    const float kLog2e = 1.4426950408889634f;
    int li = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++li) {
      const int b = li & 1;
      ok = __all_sync(0xffffffffu, wait_bar(bar(B_ACCFULL + b), (li >> 1) & 1, wc, 621));
      if (!ok) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, a.n_tm, a.n_tn, tm, tn);
      const int row = tm * kBM + r;
      const bool row_in = row < a.M;
      const uint32_t acc = tmem + lad + b * kBN;
      __nv_bfloat16* orow = a.out + static_cast<size_t>(row_in ? row : 0) * a.ldo;
      if (kEpi == EPI_SWIGLU) {
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
            uint4* dst = reinterpret_cast<uint4*>(orow + tn * 128 + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          float v32[32];
          __syncwarp();
          tmem_ld32(acc + c * 32, v32);
          if (row_in) {
            uint4* dst = reinterpret_cast<uint4*>(orow + tn * kBN + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pack_bf16x2(v32[8 * v], v32[8 * v + 1]),
                                  pack_bf16x2(v32[8 * v + 2], v32[8 * v + 3]),
                                  pack_bf16x2(v32[8 * v + 4], v32[8 * v + 5]),
                                  pack_bf16x2(v32[8 * v + 6], v32[8 * v + 7]));
          }
        }
      }
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
