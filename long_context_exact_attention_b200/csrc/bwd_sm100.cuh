// bwd_sm100.cuh -- exact attention backward, bf16, head dim 128, sm_100a.
//
// Gradients of sum(dO * O), recomputing the attention matrix from the saved
// log-sum-exp instead of storing it (the attention-level form of activation
// checkpointing the long-context recipes rely on: sourcepulse project card
// of the 1M-context recipe, How It Works).  With D_i = dO_i . O_i:
//   S^T  = K Q^T                  P^T = exp2(S^T * c - lse_i * log2 e)
//   dP^T = V dO^T                 dS^T = P^T o (dP^T - D_i)
//   dV  += P^T dO                 dK  += dS^T Q          (TMEM accumulators)
//   dQ^T = K^T dS^T -> added into the fp32 dq accumulator by TMA bulk
//                      reduce-add (scale applied later)
// Ragged and packed sequences: the rows of the last tile past the end of a
// sequence load whatever follows it on the flattened token axis (the next
// batch entry or packed sequence, zeros past the tensor's end).  Query rows
// there have an lse copy of +inf, so P and dS vanish in their columns and
// their dQ^T columns are exact zeros (the reduce-adds leave the following
// rows' accumulator unchanged); key rows there get an exponent of -inf, so
// P = 0 and dS = 0, and their dK/dV are not stored.
//
// One CTA per (key tile of 128, key/value head, batch); it loops over the
// query heads of its grouped-query group and over the query tiles that can
// see the key tile, so dK/dV of a key tile finish inside one CTA.
//
// Block calls: the key tiles belong to a key/value block that may start
// elsewhere on the position axis than the query block (a sequence-parallel
// ring; Ring Attention with Blockwise Transformers, Summary), with its own
// length and a shifted causal diagonal (AttnSched::diag).  With kAccKV the
// CTA writes its dK/dV in float32, added to what the buffers hold when
// acc_add is set (the ring carries such accumulators with the key/value
// block from host to host), instead of storing bf16.
// Roles (16 warps, four warpgroups):
//   warpgroup 0  warp 0: TMA producer (K, V once; Q + lse/D rows through a
//                2-stage ring, dO single-staged); warp 1: TMEM owner, lane 0
//                issues the five MMAs of every step; warps 2-3 idle.  The
//                warpgroup gives up registers to the other three.
//   warpgroups 1, 2  P/dS: one key row per thread, warpgroup h taking query
//                columns [64(h-1), 64h).  P^T (bf16) is written back inside
//                the S^T columns the same warpgroup read and feeds the dV
//                product straight from tensor memory; dS^T goes to shared
//                memory (an operand of both dK and dQ^T)
//   warpgroup 3  dQ: one head dim per thread; moves dQ^T from TMEM through
//                shared memory (one [64 query x 32 dim] box per warp) into
//                a TMA reduce-add of the accumulator; writes dV at the end
// TMEM: S^T then P^T [0,128) | dP^T then dQ^T [128,256) | dV | dK
#pragma once

#include "ptx.cuh"
#include "sched.cuh"

namespace lca {

namespace bwd {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr uint32_t kHalf = kTile * 64 * 2;
constexpr uint32_t kTileB = 2 * kHalf;
constexpr int kThreads = 512;
// Registers per thread at launch (launch bounds 512 x 1 CTA) and the split
// the warpgroups take with setmaxnreg: control 56, the two P/dS warpgroups
// 160 each, the dQ warpgroup 136 (56 + 2 * 160 + 136 = 4 * 128; the dQ
// warpgroup spills below 128, the control one below 56).
constexpr int kRegsLaunch = 128;
constexpr int kRegsCtl = 56;
constexpr int kRegsWork = 160;
constexpr int kRegsDq = 136;
static_assert(kRegsCtl + 2 * kRegsWork + kRegsDq == 4 * kRegsLaunch, "register split");

constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kTileB;
constexpr uint32_t kOffQ = kOffV + kTileB;        // 2 stages
constexpr uint32_t kOffO = kOffQ + 2 * kTileB;    // dO, 1 stage
constexpr uint32_t kOffS = kOffO + kTileB;        // dS^T
constexpr uint32_t kOffR = kOffS + kTileB;        // dQ staging, 4 warps x 8 KB
constexpr uint32_t kOffL = kOffR + 4 * 8192;      // lse[2][128]
constexpr uint32_t kOffD = kOffL + 1024;          // D[2][128]
constexpr uint32_t kOffBar = kOffD + 1024;
constexpr uint32_t kUsed = kOffBar + 256;
// Shared memory requested: what is used plus the slack that is left under
// the 227 KB per-CTA limit; the kernel refuses to run if aligning its base
// to 1024 bytes would need more than that slack.
constexpr uint32_t kSmemBytes = 232448;
constexpr uint32_t kSlack = kSmemBytes - kUsed;
static_assert(kUsed <= kSmemBytes, "shared memory");

enum {
  B_KV = 0,
  B_QFULL,        // +stage
  B_QEMPTY = 3,   // +stage
  B_OFULL = 5,
  B_OEMPTY,
  B_SFULL,
  B_DPFULL,
  B_PREADY,       // 256 arrivals
  B_DSREADY,      // 256 arrivals
  B_DSFREE,
  B_DQFULL,
  B_DQFREE,       // 128 arrivals
  B_DONE,
  B_DRAIN,
  NUM_BARS
};

constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
constexpr uint32_t kIdescKM = idesc_bf16_f32(128, 128, false, true);   // dV, dK
constexpr uint32_t kIdescMM = idesc_bf16_f32(128, 128, true, true);    // dQ^T

struct Args {
  int B, Hq, Hkv;
  int S;                 // tokens per batch entry of the tensors (packed: all sequences)
  int S_pad;             // row length of the padded lse / D copies
  float scale;
  float scale_log2;
  unsigned long long budget;
  const float* lse;      // [B,Hq,S_pad], +inf past each sequence's end
  const float* Drow;     // [B,Hq,S_pad], zero past each sequence's end
  __nv_bfloat16* dk;     // bf16 outputs (kAccKV false)
  __nv_bfloat16* dv;
  float* dk_acc;         // float32 accumulators, [B, S_kv, Hkv, 128] (kAccKV true)
  float* dv_acc;
  int acc_add;           // kAccKV: add to dk_acc/dv_acc (else overwrite them)
  AttnSched sched;
};

}  // namespace bwd

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <bool kAccKV>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    attn_bwd_bf16_sm100(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmDQ,
                        const __grid_constant__ bwd::Args a) {
  using namespace bwd;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (base - raw > kSlack) {
    // Cannot place the 1024-aligned layout inside the allocation: refuse.
    if (threadIdx.x == 0) record_error(kErrSmemAlign, 100);
    return;
  }
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + kOffK, sV = base + kOffV, sQ = base + kOffQ, sO = base + kOffO;
  const uint32_t sS = base + kOffS, sR = base + kOffR, sL = base + kOffL, sD = base + kOffD;
  const float* lse_s = reinterpret_cast<const float*>(gbase + kOffL);
  const float* d_s = reinterpret_cast<const float*>(gbase + kOffD);
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * NUM_BARS + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  const AttnSched& sc = a.sched;
  const int rep = a.Hq / a.Hkv;
  // Head-major order (the CTAs in flight update one or two heads' dq rows,
  // which stay in L2), longest causal work first within a head: key tile 0
  // sees every query tile.
  const int kt = static_cast<int>(blockIdx.x) % sc.n_kv_tiles;
  const int bg = static_cast<int>(blockIdx.x) / sc.n_kv_tiles;
  const int g = bg % a.Hkv;
  const int b = bg / a.Hkv;
  SeqView sv;
  if (!seq_view(sc, b, a.S, &sv)) {
    if (threadIdx.x == 0 && kt == 0) record_error(kErrSeqOffsets, 151);
    return;
  }
  if (kt >= sv.kv_n_tiles) return;  // a shorter packed sequence: no work here
  const bool shifted = head_shifted(sc, g * rep);
  const int ktok0 = token_tile(sc, kt, shifted) * kTile;
  QWalk qw;
  qw.init(&sc, kt, sv.n_tiles);
  const int nq = qw.count();
  const int nsteps = rep * nq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) {
      const uint32_t cnt = (i == B_PREADY || i == B_DSREADY) ? 256u
                           : (i == B_DQFREE)                 ? 128u
                                                             : 1u;
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

  if (wg == 0) {
    regs_dec<kRegsCtl>();
    if (warp == 0 && lane == 0) {
      // =================================================== TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(bar(B_KV), 2 * kTileB);
      const int ktok = sv.kv_row0 + ktok0;
      tma_load_3d(sK, &tmK, bar(B_KV), 0, g, ktok);
      tma_load_3d(sK + kHalf, &tmK, bar(B_KV), 64, g, ktok);
      tma_load_3d(sV, &tmV, bar(B_KV), 0, g, ktok);
      tma_load_3d(sV + kHalf, &tmV, bar(B_KV), 64, g, ktok);
      bool ok = true;
      int issued0 = 0, issued1 = 0, o_issued = 0;
      for (int i = 0; i < nsteps && ok; ++i) {
        const int st = i & 1;
        const int h = g * rep + i / nq;
        const int qt = qw.t + i % nq;
        const int qtok0 = token_tile(sc, qt, shifted) * kTile;
        if (i >= 2) ok = wait_bar(bar(B_QEMPTY + st), ((i - 2) >> 1) & 1, wc, 111);
        if (!ok) break;
        const uint32_t fb = bar(B_QFULL + st);
        mbar_expect_tx(fb, kTileB + 1024);
        tma_load_3d(sQ + st * kTileB, &tmQ, fb, 0, h, sv.row0 + qtok0);
        tma_load_3d(sQ + st * kTileB + kHalf, &tmQ, fb, 64, h, sv.row0 + qtok0);
        const size_t ro = (static_cast<size_t>(b) * a.Hq + h) * a.S_pad + qtok0;
        bulk_load(sL + st * 512, a.lse + ro, 512, fb);
        bulk_load(sD + st * 512, a.Drow + ro, 512, fb);
        if (st) ++issued1; else ++issued0;
        if (i >= 1) ok = wait_bar(bar(B_OEMPTY), (i - 1) & 1, wc, 112);
        if (!ok) break;
        mbar_expect_tx(bar(B_OFULL), kTileB);
        tma_load_3d(sO, &tmDO, bar(B_OFULL), 0, h, sv.row0 + qtok0);
        tma_load_3d(sO + kHalf, &tmDO, bar(B_OFULL), 64, h, sv.row0 + qtok0);
        ++o_issued;
      }
      if (!ok) {
        drain_bar(bar(B_KV), 0, 171);
        if (issued0) drain_bar(bar(B_QFULL), (issued0 - 1) & 1, 172);
        if (issued1) drain_bar(bar(B_QFULL + 1), (issued1 - 1) & 1, 173);
        if (o_issued) drain_bar(bar(B_OFULL), (o_issued - 1) & 1, 174);
      }
    } else if (warp == 1 && lane == 0) {
      // =================================================== MMA issuer
      // Order per step i: dP^T_i, dV_i, S^T_{i+1}, dK_i, dQ^T_i.  S^T_{i+1}
      // goes right behind dV_i, the last reader of the S^T/P^T columns (the
      // tensor pipe runs this thread's MMAs in order), so the next step's
      // P phase overlaps dK_i and dQ^T_i.
      const uint32_t tSt = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
      auto issue_s = [&](int i) {
        const uint32_t q_s = sQ + (i & 1) * kTileB;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          mma_bf16_ss(tSt, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(q_s + off, 16, 1024),
                      kIdescKK, k > 0);
        }
        tc_commit(bar(B_SFULL));
      };
      bool ok = wait_bar(bar(B_KV), 0, wc, 211);
      if (ok && nsteps > 0) ok = wait_bar(bar(B_QFULL), 0, wc, 212);
      if (ok && nsteps > 0) {
        tc_fence_after();
        issue_s(0);
      }
      for (int i = 0; i < nsteps && ok; ++i) {
        const int st = i & 1;
        const uint32_t q_s = sQ + st * kTileB;
        ok = wait_bar(bar(B_OFULL), i & 1, wc, 214);
        if (ok && i >= 1) ok = wait_bar(bar(B_DQFREE), (i - 1) & 1, wc, 215);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          mma_bf16_ss(tdP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sO + off, 16, 1024),
                      kIdescKK, k > 0);
        }
        tc_commit(bar(B_DPFULL));
        ok = wait_bar(bar(B_PREADY), i & 1, wc, 216);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO, P^T read from tensor memory: queries [0,64) at columns
        // [0,32), queries [64,128) at [64,96), 8 columns per 16 queries
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mma_bf16_ts(tdV, tSt + (k >> 2) * 64 + (k & 3) * 8,
                      sdesc_sw128(sO + k * 2048, kHalf, 1024), kIdescKM, (i > 0 || k > 0));
        }
        tc_commit(bar(B_OEMPTY));
        if (i + 1 < nsteps) {
          ok = wait_bar(bar(B_QFULL + (st ^ 1)), ((i + 1) >> 1) & 1, wc, 213);
          if (!ok) break;
          tc_fence_after();
          issue_s(i + 1);
        }
        ok = wait_bar(bar(B_DSREADY), i & 1, wc, 217);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t offa = (k >> 2) * kHalf + (k & 3) * 32;
          mma_bf16_ss(tdK, sdesc_sw128(sS + offa, 16, 1024),
                      sdesc_sw128(q_s + k * 2048, kHalf, 1024), kIdescKM, (i > 0 || k > 0));
        }
        tc_commit(bar(B_QEMPTY + st));
        // dQ^T = K^T dS^T: A = K (head dims contiguous), B = dS^T (queries
        // contiguous), both MN-major; K steps of 16 keys
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mma_bf16_ss(tdP, sdesc_sw128(sK + k * 2048, kHalf, 1024),
                      sdesc_sw128(sS + k * 2048, kHalf, 1024), kIdescMM, k > 0);
        }
        tc_commit(bar(B_DQFULL));
        tc_commit(bar(B_DSFREE));
      }
      tc_commit(bar(B_DONE));
      tc_commit(bar(B_DRAIN));
      drain_bar(bar(B_DRAIN), 0, 175);
    }
  } else if (wg <= 2) {
    regs_inc<kRegsWork>();
    // =================================================== P / dS warpgroups
    const int hq = wg - 1;             // query-column half of this warpgroup
    const int wq = warp & 3;
    const int r = wq * 32 + lane;      // key row
    const uint32_t lad = static_cast<uint32_t>(wq * 32) << 16;
    const float c = a.scale_log2;
    const float L2E = 1.4426950408889634f;
    const uint64_t c2 = f2_pack(c, c);
    const bool key_out = ktok0 + r >= sv.kv_len;  // key row past the sequence's end
    // added to every exponent of this key row: -inf gives P = 0 (hence dS =
    // 0, and the row adds nothing to dQ) for a key row past the end
    const float kill = key_out ? -INFINITY : 0.f;
    bool ok = true;
    for (int i = 0; i < nsteps && ok; ++i) {
      const int st = i & 1;
      const int qt = qw.t + i % nq;
      const float* lse_r = lse_s + st * 128 + hq * 64;
      const float* d_r = d_s + st * 128 + hq * 64;
      ok = wait_bar(bar(B_SFULL), i & 1, wc, 311);
      if (ok) ok = wait_bar(bar(B_QFULL + st), (i >> 1) & 1, wc, 312);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool diag = sc.causal && qt + sc.diag == kt;
      // ---- P^T = exp2(S^T c - lse log2e) for queries [64hq, 64hq+64),
      // written back as bf16 over columns [64hq, 64hq+32) of S^T
      float p[64];
      tmem_ld64(tmem + lad + hq * 64, p);
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const int q0 = hq * 64 + e;
          const uint64_t nl =
              f2_pack(fmaf(-lse_r[e], L2E, kill), fmaf(-lse_r[e + 1], L2E, kill));
          float p0, p1;
          f2_unpack(f2_fma(f2_pack(p[e], p[e + 1]), c2, nl), p0, p1);
          p0 = ex2_approx(p0);
          p1 = ex2_approx(p1);
          if (diag && r > q0) p0 = 0.f;
          if (diag && r > q0 + 1) p1 = 0.f;
          p[e] = p0;
          p[e + 1] = p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st32u(tmem + lad + hq * 64, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY));
      // ---- dS^T = P^T o (dP^T - D) -> shared memory
      ok = wait_bar(bar(B_DPFULL), i & 1, wc, 313);
      if (ok && i >= 1) ok = wait_bar(bar(B_DSFREE), (i - 1) & 1, wc, 314);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float dp[64];
      tmem_ld64(tmem + lad + 128 + hq * 64, dp);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int ql = cc * 32 + e;
          const uint64_t t = f2_sub(f2_pack(dp[ql], dp[ql + 1]), f2_pack(d_r[ql], d_r[ql + 1]));
          float t0, t1;
          f2_unpack(t, t0, t1);
          dd[e >> 1] = pack_bf16x2(p[ql] * t0, p[ql + 1] * t1);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int cw = cc * 4 + v;  // 16-byte chunk within this half's 128-byte row
          const uint32_t off = hq * kHalf + r * 128 + ((cw ^ (r & 7)) << 4);
          st_shared_v4(sS + off, dd[4 * v], dd[4 * v + 1], dd[4 * v + 2], dd[4 * v + 3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_DSREADY));
    }
    // ---- dK = scale * acc -> bf16 (columns split between the two halves)
    if (ok) ok = wait_bar(bar(B_DONE), 0, wc, 315);
    ok = __all_sync(0xffffffffu, ok);
    // every lane takes part in the TMEM loads (warp-collective); key rows
    // past the sequence's end (ragged last tile) only skip their stores
    if (ok) {
      tc_fence_after();
      const size_t trow = static_cast<size_t>(sv.kv_row0) + (key_out ? 0 : ktok0 + r);
      __nv_bfloat16* row = a.dk + (trow * a.Hkv + g) * kD;
      float* arow = a.dk_acc + (trow * a.Hkv + g) * kD;
#pragma unroll 1
      for (int cc = 2 * hq; cc < 2 * hq + 2; ++cc) {
        float o[32];
        __syncwarp();
        if (nsteps > 0) {
          tmem_ld32(tmem + lad + 384 + cc * 32, o);
        } else {  // a block call's key tile that no query sees: no gradient
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (kAccKV && !key_out) {
          float4* dst = reinterpret_cast<float4*>(arow + cc * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 x = a.acc_add ? dst[v] : make_float4(0.f, 0.f, 0.f, 0.f);
            dst[v] = make_float4(fmaf(o[4 * v], a.scale, x.x), fmaf(o[4 * v + 1], a.scale, x.y),
                                 fmaf(o[4 * v + 2], a.scale, x.z),
                                 fmaf(o[4 * v + 3], a.scale, x.w));
          }
        } else if (!key_out) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pk;
            pk.x = pack_bf16x2(o[v * 8 + 0] * a.scale, o[v * 8 + 1] * a.scale);
            pk.y = pack_bf16x2(o[v * 8 + 2] * a.scale, o[v * 8 + 3] * a.scale);
            pk.z = pack_bf16x2(o[v * 8 + 4] * a.scale, o[v * 8 + 5] * a.scale);
            pk.w = pack_bf16x2(o[v * 8 + 6] * a.scale, o[v * 8 + 7] * a.scale);
            *reinterpret_cast<uint4*>(row + cc * 32 + v * 8) = pk;
          }
        }
      }
    }
  } else {
    regs_inc<kRegsDq>();
    // =================================================== dQ warpgroup
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // head dim (dQ^T) / key row (dV)
    const uint32_t lad = static_cast<uint32_t>(wq * 32) << 16;
    // this warp's staging box: [64 queries][32 head dims] fp32, rows of 128 B
    const uint32_t stage = sR + wq * 8192 + lane * 4;
    if (lane == 0) tma_prefetch_desc(&tmDQ);
    bool ok = true;
    for (int i = 0; i < nsteps && ok; ++i) {
      const int h = g * rep + i / nq;
      const int qt = qw.t + i % nq;
      const int qtok0 = token_tile(sc, qt, shifted) * kTile;
      ok = __all_sync(0xffffffffu, wait_bar(bar(B_DQFULL), i & 1, wc, 411));
      if (!ok) break;
      tc_fence_after();
      float dq0[64], dq1[64];
      tmem_ld64(tmem + lad + 128, dq0);
      tmem_ld64(tmem + lad + 192, dq1);
      tc_fence_before();
      mbar_arrive(bar(B_DQFREE));
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // the previous reduce from this buffer must have read it
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage + q * 128),
                       "f"(half ? dq1[q] : dq0[q])
                       : "memory");
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmDQ, sR + wq * 8192, wq * 32, h, sv.row0 + qtok0 + half * 64);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
    // ---- dV -> bf16
    if (ok) ok = wait_bar(bar(B_DONE), 0, wc, 412);
    ok = __all_sync(0xffffffffu, ok);
    const bool row_in = ktok0 + r < sv.kv_len;
    if (ok) {
      tc_fence_after();
      const size_t trow = static_cast<size_t>(sv.kv_row0) + (row_in ? ktok0 + r : 0);
      __nv_bfloat16* row = a.dv + (trow * a.Hkv + g) * kD;
      float* arow = a.dv_acc + (trow * a.Hkv + g) * kD;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float o[32];
        __syncwarp();
        if (nsteps > 0) {
          tmem_ld32(tmem + lad + 256 + cc * 32, o);
        } else {  // a block call's key tile that no query sees: no gradient
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (kAccKV && row_in) {
          float4* dst = reinterpret_cast<float4*>(arow + cc * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 x = a.acc_add ? dst[v] : make_float4(0.f, 0.f, 0.f, 0.f);
            dst[v] = make_float4(o[4 * v] + x.x, o[4 * v + 1] + x.y, o[4 * v + 2] + x.z,
                                 o[4 * v + 3] + x.w);
          }
        } else if (row_in) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pk;
            pk.x = pack_bf16x2(o[v * 8 + 0], o[v * 8 + 1]);
            pk.y = pack_bf16x2(o[v * 8 + 2], o[v * 8 + 3]);
            pk.z = pack_bf16x2(o[v * 8 + 4], o[v * 8 + 5]);
            pk.w = pack_bf16x2(o[v * 8 + 6], o[v * 8 + 7]);
            *reinterpret_cast<uint4*>(row + cc * 32 + v * 8) = pk;
          }
        }
      }
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
