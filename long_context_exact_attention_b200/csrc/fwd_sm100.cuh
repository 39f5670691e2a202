// fwd_sm100.cuh -- exact attention forward, bf16, head dim 128, sm_100a.
//
// One CTA per (query tile of 128 rows, query head, batch).  Roles:
//   warp 0      TMA producer: Q once, then K and V tiles through 2-stage rings
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma
//   warps 2..5  softmax warpgroup, one query row per thread (TMEM lane)
//
// Per key/value tile j (Ring Attention with Blockwise Transformers,
// Summary: each query block is attended block by block):
//   S_j = Q K_j^T                      tcgen05, bf16 x bf16 -> fp32 in TMEM
//   m   = running row max (log2 domain, scale folded in)
//   P_j = exp2(S_j*c - m)  -> bf16 -> swizzled shared memory
//   O  += P_j V_j                      tcgen05, fp32 accumulator in TMEM
// with the running (m, l, O) rescaled by exp2(m_old - m_new) whenever the
// running max moves by more than 8 (log2 units).  Keeping a stale max within
// that margin is exact: numerator and denominator share it, and P stays
// below 2^8.  Moving from one key chunk to the next is the (O, lse) merge of
// the summary in unnormalised form -- the same rescale.
//
// TMEM columns: S buffer 0 = [0,128), S buffer 1 = [128,256), O = [256,384).
// Shared memory (1024-aligned, 128-byte swizzle everywhere):
//   Q 32 KB | K stage 0,1 (32 KB each) | V stage 0,1 | P 32 KB | barriers
// Each 128x128 bf16 tile is two 16 KB halves (head dims 0-63, 64-127, or
// keys 0-63, 64-127 for P), rows of 128 bytes.
#pragma once

#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace lca {

namespace fwd {

// Pairs q (of the 64 per row and tile) with bit (q % 8) set would take the
// FMA-pipe polynomial exp2 instead of ex2.approx.  Measured on B200 the
// mixes tried (3/8, 4/8) were slower than none, so none is used.
constexpr uint32_t kPolyPairs = 0u;

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr uint32_t kHalf = kTile * 64 * 2;  // 16 KB
constexpr uint32_t kTileB = 2 * kHalf;      // 32 KB
constexpr int kThreads = 192;

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileB;          // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileB;      // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTileB;
constexpr uint32_t kOffBar = kOffP + kTileB;        // barriers (8 B each)
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack

// barrier indices
enum {
  B_Q = 0,
  B_KFULL = 1,   // +stage
  B_KEMPTY = 3,  // +stage
  B_VFULL = 5,   // +stage
  B_VEMPTY = 7,  // +stage
  B_SFULL = 9,   // +buffer
  B_SFREE = 11,  // +buffer
  B_PFULL = 13,
  B_OREADY = 14,
  B_DRAIN = 15,
  NUM_BARS = 16
};

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q K^T
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, false, true);    // P V (V MN-major)

struct Args {
  int B, Hq, Hkv, S;
  float scale_log2;
  unsigned long long budget;
  __nv_bfloat16* out;
  float* lse;
  AttnSched sched;
};

}  // namespace fwd

__global__ void __launch_bounds__(fwd::kThreads, 1)
    attn_fwd_bf16_sm100(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ fwd::Args a) {
  using namespace fwd;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV, sP = base + kOffP;
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * NUM_BARS + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: longest causal tiles first, heads of one tile adjacent
  const AttnSched& sc = a.sched;
  const int BH = a.B * a.Hq;
  const int qt = sc.n_tiles - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const bool shifted = head_shifted(sc, h);
  const int q_tok0 = token_tile(sc, qt, shifted) * kTile;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) {
      uint32_t cnt = 1;
      if (i == B_SFREE || i == B_SFREE + 1 || i == B_PFULL) cnt = 128;
      mbar_init(bar(i), cnt);
    }
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
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int row0 = b * a.S;
      mbar_expect_tx(bar(B_Q), kTileB);
      tma_load_3d(sQ, &tmQ, bar(B_Q), 0, h, row0 + q_tok0);
      tma_load_3d(sQ + kHalf, &tmQ, bar(B_Q), 64, h, row0 + q_tok0);
      KvWalk w;
      w.init(&sc, qt);
      int t, j = 0;
      int k_issued0 = 0, k_issued1 = 0, v_issued0 = 0, v_issued1 = 0;
      bool ok = true;
      while (ok && w.next(t)) {
        const int st = j & 1;
        const int tok = row0 + token_tile(sc, t, shifted) * kTile;
        if (j >= 2) ok = wait_bar(bar(B_KEMPTY + st), ((j - 2) >> 1) & 1, wc, 101);
        if (!ok) break;
        mbar_expect_tx(bar(B_KFULL + st), kTileB);
        tma_load_3d(sK + st * kTileB, &tmK, bar(B_KFULL + st), 0, g, tok);
        tma_load_3d(sK + st * kTileB + kHalf, &tmK, bar(B_KFULL + st), 64, g, tok);
        if (st) ++k_issued1; else ++k_issued0;
        if (j >= 2) ok = wait_bar(bar(B_VEMPTY + st), ((j - 2) >> 1) & 1, wc, 102);
        if (!ok) break;
        mbar_expect_tx(bar(B_VFULL + st), kTileB);
        tma_load_3d(sV + st * kTileB, &tmV, bar(B_VFULL + st), 0, g, tok);
        tma_load_3d(sV + st * kTileB + kHalf, &tmV, bar(B_VFULL + st), 64, g, tok);
        if (st) ++v_issued1; else ++v_issued0;
        ++j;
      }
      if (!ok) {
        // Unwind: let the copies already issued land before the CTA exits.
        drain_bar(bar(B_Q), 0, a.budget);
        if (k_issued0) drain_bar(bar(B_KFULL), (k_issued0 - 1) & 1, a.budget);
        if (k_issued1) drain_bar(bar(B_KFULL + 1), (k_issued1 - 1) & 1, a.budget);
        if (v_issued0) drain_bar(bar(B_VFULL), (v_issued0 - 1) & 1, a.budget);
        if (v_issued1) drain_bar(bar(B_VFULL + 1), (v_issued1 - 1) & 1, a.budget);
      }
    }
  } else if (warp == 1) {
    // =================================================== MMA issuer
    if (lane == 0) {
      const uint32_t tS = tmem;          // + 128 * buffer
      const uint32_t tO = tmem + 256;
      bool ok = wait_bar(bar(B_Q), 0, wc, 201);
      KvWalk w;
      w.init(&sc, qt);
      int t, j = 0;
      auto issue_pv = [&](int jj) -> bool {
        if (!wait_bar(bar(B_PFULL), jj & 1, wc, 204)) return false;
        if (!wait_bar(bar(B_VFULL + (jj & 1)), (jj >> 1) & 1, wc, 205)) return false;
        tc_fence_after();
        const uint32_t vbase = sV + (jj & 1) * kTileB;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = sdesc_sw128(sP + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(vbase + k * 2048, kHalf, 1024);
          mma_bf16_ss(tO, ad, bd, kIdescO, (jj > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_OREADY));
        tc_commit(bar(B_VEMPTY + (jj & 1)));
        return true;
      };
      while (ok && w.next(t)) {
        const int st = j & 1;
        ok = wait_bar(bar(B_KFULL + st), (j >> 1) & 1, wc, 202);
        if (!ok) break;
        if (j >= 2) ok = wait_bar(bar(B_SFREE + st), ((j - 2) >> 1) & 1, wc, 203);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sK + st * kTileB;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          const uint64_t ad = sdesc_sw128(sQ + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(kbase + off, 16, 1024);
          mma_bf16_ss(tS + st * 128, ad, bd, kIdescS, k > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + st));
        tc_commit(bar(B_KEMPTY + st));
        if (j >= 1) ok = issue_pv(j - 1);
        ++j;
      }
      if (ok && j >= 1) ok = issue_pv(j - 1);
      // Drain: wait for every MMA this thread issued before TMEM is freed.
      tc_commit(bar(B_DRAIN));
      drain_bar(bar(B_DRAIN), 0, a.budget);
    }
  } else {
    // =================================================== softmax warpgroup
    const int wq = warp & 3;             // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;        // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_addr;
    const uint32_t tO = tmem + lane_addr + 256;
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    KvWalk w;
    w.init(&sc, qt);
    int t, j = 0;
    bool ok = true;
    while (ok && w.next(t)) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, wait_bar(bar(B_SFULL + st), (j >> 1) & 1, wc, 301));
      if (!ok) break;
      tc_fence_after();
      float s[128];
      tmem_ld128(tS + st * 128, s);
      tc_fence_before();
      mbar_arrive(bar(B_SFREE + st));
      const bool diag = sc.causal && (t == qt);
      if (diag) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > r) s[i] = -INFINITY;
      }
      // Row max: eight independent chains of 3-input max.
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
      for (int i = 16; i < 128; i += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], s[i + 2 * k], s[i + 2 * k + 1]);
      }
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
      const float m_cand = fmaxf(m_run, mx * c);
      const float m_new = (m_cand > m_run + 8.0f || m_run == -INFINITY) ? m_cand : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_use);
      // P = 2^(s*c - m) in pairs; off the diagonal 3 of every 8 pairs go
      // through the FMA-pipe polynomial, the rest through ex2.approx.
      uint32_t pk[64];
      uint64_t acc[4] = {0, 0, 0, 0};
      const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
      if (diag) {
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          float a, b;
          f2_unpack(f2_fma(f2_pack(s[2 * q], s[2 * q + 1]), c2, nm2), a, b);
          a = ex2_approx(a);
          b = ex2_approx(b);
          acc[q & 3] = f2_add(acc[q & 3], f2_pack(a, b));
          pk[q] = pack_bf16x2(a, b);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          const uint64_t x = f2_fma(f2_pack(s[2 * q], s[2 * q + 1]), c2, nm2);
          float a, b;
          if ((kPolyPairs >> (q & 7)) & 1u) {
            f2_unpack(exp2_poly_x2(x), a, b);
          } else {
            f2_unpack(x, a, b);
            a = ex2_approx(a);
            b = ex2_approx(b);
          }
          acc[q & 3] = f2_add(acc[q & 3], f2_pack(a, b));
          pk[q] = pack_bf16x2(a, b);
        }
      }
      float rsum;
      {
        const uint64_t t01 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float lo, hi;
        f2_unpack(t01, lo, hi);
        rsum = lo + hi;
      }
      l_run = l_run * alpha + rsum;
      m_run = m_new;
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_OREADY), (j - 1) & 1, wc, 302));
        if (!ok) break;
        tc_fence_after();
        // Rescale the O row when the running max moved (warp-uniform ld/st).
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(tO + cc * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + cc * 32, o);
          }
          tmem_st_wait();
        }
      }
      // P (bf16) -> shared memory, 128-byte swizzle, K-major rows of keys.
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int half = ch >> 3, cw = ch & 7;
        const uint32_t addr = sP + half * kHalf + r * 128 + ((cw ^ (r & 7)) << 4);
        st_shared_v4(addr, pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL));
      ++j;
    }
    // ---- epilogue: O / l -> bf16 out, lse = ln(2) * (m + log2 l)
    if (ok && j >= 1) ok = wait_bar(bar(B_OREADY), (j - 1) & 1, wc, 303);
    ok = __all_sync(0xffffffffu, ok && j >= 1);
    const int tok = q_tok0 + r;
    if (ok) {
      tc_fence_after();
      const float inv = (l_run > 0.f) ? 1.0f / l_run : 0.f;
      __nv_bfloat16* orow =
          a.out + ((static_cast<size_t>(b) * a.S + tok) * a.Hq + h) * kD;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float o[32];
        tmem_ld32(tO + cc * 32, o);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 pk;
          pk.x = pack_bf16x2(o[v * 8 + 0] * inv, o[v * 8 + 1] * inv);
          pk.y = pack_bf16x2(o[v * 8 + 2] * inv, o[v * 8 + 3] * inv);
          pk.z = pack_bf16x2(o[v * 8 + 4] * inv, o[v * 8 + 5] * inv);
          pk.w = pack_bf16x2(o[v * 8 + 6] * inv, o[v * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(orow + cc * 32 + v * 8) = pk;
        }
      }
      const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f
                                      : -INFINITY;
      a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.S + tok] = lse;
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
