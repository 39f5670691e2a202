// fwd2_sm100.cuh -- exact attention forward on CTA pairs (tcgen05
// cta_group::2), bf16, head dimension 128, sm_100a.
//
// Same computation as attn_fwd_bf16_sm100 (fwd_sm100.cuh): per key/value
// tile, S = Q K^T, the online softmax with the lazy rescale, O += P V, the
// (O, lse) merge of chunks in unnormalised form.  What changes is how the
// tensor cores are fed.  With one CTA the product S = Q K^T takes both
// operands from shared memory, 64 KB per 128x128x128 product -- exactly the
// shared-memory bandwidth of an SM while the tensor pipe runs at full rate,
// so the forward was bound three ways at once (tensor pipe, exponentials,
// shared memory).  Here two CTAs on neighbouring SMs form a pair and issue
// M = 256 products: each CTA supplies its own 128 query rows and HALF of
// the key tile (64 keys) for S = Q K^T, and half of the value tile (64 of
// the head dimensions) for O += P V; the pair's tensor cores exchange the
// halves.  Per key tile and CTA the shared-memory traffic falls from 256 KB
// to 160 KB (operands 128 KB -> 96 KB, TMA writes 64 KB -> 32 KB).
//
// Work item of a pair: four consecutive query tiles 4u .. 4u+3 of one head;
// CTA c owns tiles 4u + c and 4u + 2 + c, so the pair's product for query
// slot t covers tiles 4u + 2t (CTA 0) and 4u + 2t + 1 (CTA 1), one diagonal
// apart.  A key tile that only the later of the two sees still runs the
// pair product; the other CTA writes P = 0 for it.  Both CTAs walk the key
// tiles of the quad's last tile, in the chunk order of the schedule.
//
// Roles in each CTA: warp 0 TMA producer (own Q tiles once, own halves of
// K and V through a 3-stage ring; completion counted on the leader's
// barriers); warp 1 TMEM owner, and in the leader (rank 0) lane 0 issues
// every pair MMA; warps 2-5 / 6-9 softmax of query slot 0 / 1, one row per
// thread, P written back into S's TMEM columns; their arrivals go to the
// leader's barrier.  The leader's commits arrive on both CTAs' barriers.
//
// No TMA load here multicasts; every load writes only its own CTA's shared
// memory from global memory.
#pragma once

#include "fwd_sm100.cuh"

namespace lca {

namespace fwd2 {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr uint32_t kQHalf = kTile * 64 * 2;   // 16 KB: 128 rows x 64 dims
constexpr uint32_t kQTile = 2 * kQHalf;       // 32 KB
constexpr uint32_t kKBox = 64 * 64 * 2;       // 8 KB: 64 keys x 64 dims
constexpr uint32_t kKStage = 2 * kKBox;       // 16 KB: this CTA's 64 keys x 128 dims
constexpr uint32_t kVStage = kTile * 64 * 2;  // 16 KB: 128 keys x this CTA's 64 dims
constexpr int kStages = 3;
constexpr int kThreads = 320;

constexpr uint32_t kOffQ = 0;                            // 2 query tiles
constexpr uint32_t kOffK = kOffQ + 2 * kQTile;           // kStages
constexpr uint32_t kOffV = kOffK + kStages * kKStage;    // kStages
constexpr uint32_t kOffBar = kOffV + kStages * kVStage;  // barriers (8 B each)
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;    // + alignment slack

enum {
  // counted on the leader's copy: both producers (expect_tx) / both CTAs'
  // softmax threads arrive there
  L_Q = 0,
  L_KFULL = 1,                    // + stage
  L_VFULL = L_KFULL + kStages,    // + stage
  L_PFULL = L_VFULL + kStages,    // + query slot, 256 arrivals
  // every CTA's own copy, arrived on by the leader's commits
  B_KEMPTY = L_PFULL + 2,         // + stage
  B_VEMPTY = B_KEMPTY + kStages,  // + stage
  B_SFULL = B_VEMPTY + kStages,   // + query slot
  B_OREADY = B_SFULL + 2,         // + query slot
  B_DRAIN = B_OREADY + 2,
  NUM_BARS
};
static_assert(NUM_BARS * 8 + 64 <= 512, "barrier area");

constexpr uint32_t kIdescS = idesc_bf16_f32(256, 128, false, false);  // Q K^T
constexpr uint32_t kIdescO = idesc_bf16_f32(256, 128, false, true);   // P V (V MN-major)

}  // namespace fwd2

// kBlock: a block call (merging epilogue), as attn_fwd_bf16_sm100.  Only the
// tile walk (chunks of whole tiles) runs here.
template <bool kBlock>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(fwd2::kThreads, 1)
    attn_fwd_bf16_sm100_pair(const __grid_constant__ CUtensorMap tmQ,
                             const __grid_constant__ CUtensorMap tmK,   // box of 64 keys
                             const __grid_constant__ CUtensorMap tmV,   // box of 128 keys
                             const __grid_constant__ fwd::Args a) {
  using namespace fwd2;
  using fwd::VIS_DIAG;
  using fwd::VIS_NONE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * NUM_BARS + 8);
  // [0] len, [4] row0, [8] lse offset (64-bit), [16] kv_len
  const uint32_t seq_smem = bars + 8 * NUM_BARS + 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank();
  const bool leader = crank == 0;

  // ---- work item of the pair: four query tiles, head-major, longest first
  const AttnSched& sc = a.sched;
  const int n_quads = (sc.n_tiles + 3) >> 2;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int u = n_quads - 1 - pair % n_quads;
  const int bh = pair / n_quads;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const bool shifted = head_shifted(sc, h);
  SeqView sv;
  if (!seq_view(sc, b, a.S, &sv)) {  // pair-uniform: both CTAs leave here
    if (threadIdx.x == 0 && u == 0 && leader) record_error(kErrSeqOffsets, 152);
    return;
  }
  const int q_base = 4 * u;
  if (q_base >= sv.n_tiles) return;  // pair-uniform
  // the quad's last existing tile sets the walk (it sees every key tile
  // any of the four sees)
  const int qt_last = (q_base + 3 < sv.n_tiles) ? q_base + 3 : sv.n_tiles - 1;
  const bool causal = sc.causal != 0;
  const int diag = kBlock ? sc.diag : 0;
  // this CTA's tiles per query slot, and whether they exist
  const int my_q[2] = {q_base + static_cast<int>(crank), q_base + 2 + static_cast<int>(crank)};
  // the later tile of each slot's pair (CTA 1's, or CTA 0's when it is the
  // last tile of the sequence): a slot's product runs when that tile sees T
  auto slot_last = [&](int tq) {
    const int t1 = q_base + 2 * tq + 1;
    return t1 < sv.n_tiles ? t1 : q_base + 2 * tq;
  };
  auto slot_exists = [&](int tq) { return q_base + 2 * tq < sv.n_tiles; };
  auto act = [&](int tq, int T) {
    return slot_exists(tq) && fwd::tile_vis(causal, diag, slot_last(tq), T) != VIS_NONE;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) {
      uint32_t cnt = 1;
      if (i == L_Q || (i >= L_KFULL && i < L_PFULL)) cnt = 2;
      if (i == L_PFULL || i == L_PFULL + 1) cnt = 256;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    int* si = reinterpret_cast<int*>(gbase + kOffBar + 8 * NUM_BARS + 16);
    si[0] = sv.len;
    si[1] = sv.row0;
    *reinterpret_cast<long long*>(si + 2) =
        (static_cast<long long>(sv.bm) * a.Hq + h) * a.S + sv.tokb;
    si[4] = sv.kv_len;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtl wc{abort_flag, a.budget};
  auto lbar = [&](int i) { return mapa_shared(bar(i), 0); };  // the leader's copy

  if (warp == 0) {
    // =================================================== TMA producer (each CTA)
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t qbytes = 0;
      for (int t = 0; t < 2; ++t)
        if (my_q[t] < sv.n_tiles) qbytes += kQTile;
      mbar_expect_tx_cluster(lbar(L_Q), qbytes);
      for (int t = 0; t < 2; ++t) {
        if (my_q[t] >= sv.n_tiles) continue;  // never read: that slot's P is zero here
        const int tok = sv.row0 + token_tile(sc, my_q[t], shifted) * kTile;
        tma_load_3d_pair(sQ + t * kQTile, &tmQ, lbar(L_Q), 0, h, tok);
        tma_load_3d_pair(sQ + t * kQTile + kQHalf, &tmQ, lbar(L_Q), 64, h, tok);
      }
      TileWalk w;
      w.init(&sc, qt_last, sv.kv_n_tiles);
      int t, j = 0;
      bool ok = true;
      const int koff = 64 * static_cast<int>(crank);  // this CTA's keys / head dims
      while (ok && w.next(t)) {
        const int st = j % kStages;
        const uint32_t ph = ((j / kStages) - 1) & 1;
        const int tok = sv.kv_row0 + token_tile(sc, t, shifted) * kTile;
        if (j >= kStages) ok = wait_bar(bar(B_KEMPTY + st), ph, wc, 121);
        if (!ok) break;
        mbar_expect_tx_cluster(lbar(L_KFULL + st), kKStage);
        tma_load_3d_pair(sK + st * kKStage, &tmK, lbar(L_KFULL + st), 0, g, tok + koff);
        tma_load_3d_pair(sK + st * kKStage + kKBox, &tmK, lbar(L_KFULL + st), 64, g, tok + koff);
        if (j >= kStages) ok = wait_bar(bar(B_VEMPTY + st), ph, wc, 122);
        if (!ok) break;
        mbar_expect_tx_cluster(lbar(L_VFULL + st), kVStage);
        tma_load_3d_pair(sV + st * kVStage, &tmV, lbar(L_VFULL + st), koff, g, tok);
        ++j;
      }
      // On an abort the copies already issued complete on the leader's
      // barriers; the leader drains its own MMAs, and the pair meets at the
      // closing cluster barrier only after every bounded wait has ended.
    }
  } else if (warp == 1) {
    // =================================================== pair MMA issuer (leader)
    if (leader && lane == 0) {
      bool ok = wait_bar(bar(L_Q), 0, wc, 221);
      TileWalk w;
      w.init(&sc, qt_last, sv.kv_n_tiles);
      int T, Tn;
      int pv_cnt[2] = {0, 0};
      auto issue_s = [&](int tq, int j) {
        const uint32_t kbase = sK + (j % kStages) * kKStage;
        const uint32_t qbase = sQ + tq * kQTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mma_pair_ss(tmem + tq * 128,
                      sdesc_sw128(qbase + (k >> 2) * kQHalf + (k & 3) * 32, 16, 1024),
                      sdesc_sw128(kbase + (k >> 2) * kKBox + (k & 3) * 32, 16, 1024), kIdescS,
                      k > 0 ? 1u : 0u);
        }
        tc_commit_pair(bar(B_SFULL + tq), 0x3);
      };
      bool have = ok && w.next(T);
      if (have) {
        ok = wait_bar(bar(L_KFULL), 0, wc, 222);
        if (ok) {
          tc_fence_after();
          if (act(0, T)) issue_s(0, 0);
          if (act(1, T)) issue_s(1, 0);
          tc_commit_pair(bar(B_KEMPTY), 0x3);
        }
      }
      int j = 0;
      while (ok && have) {
        const bool has_next = w.next(Tn);
        const int st = j % kStages, stn = (j + 1) % kStages;
        ok = wait_bar(bar(L_VFULL + st), (j / kStages) & 1, wc, 223);
        if (ok && has_next) ok = wait_bar(bar(L_KFULL + stn), ((j + 1) / kStages) & 1, wc, 224);
        for (int tq = 0; tq < 2 && ok; ++tq) {
          if (act(tq, T)) {
            ok = wait_bar(bar(L_PFULL + tq), pv_cnt[tq] & 1, wc, 225);
            if (!ok) break;
            tc_fence_after();
            const uint32_t vbase = sV + st * kVStage;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              mma_pair_ts(tmem + 256 + tq * 128, tmem + tq * 128 + k * 8,
                          sdesc_sw128(vbase + k * 2048, kVStage, 1024), kIdescO,
                          (pv_cnt[tq] > 0 || k > 0) ? 1u : 0u);
            }
            tc_commit_pair(bar(B_OREADY + tq), 0x3);
            ++pv_cnt[tq];
          }
          if (has_next && act(tq, Tn)) issue_s(tq, j + 1);
        }
        if (!ok) break;
        tc_commit_pair(bar(B_VEMPTY + st), 0x3);
        if (has_next) tc_commit_pair(bar(B_KEMPTY + stn), 0x3);
        have = has_next;
        T = Tn;
        ++j;
      }
      // every pair MMA done before the pair's tensor memory is freed
      tc_commit_pair(bar(B_DRAIN), 0x1);
      drain_bar(bar(B_DRAIN), 0, 167);
    }
  } else {
    // =================================================== softmax warpgroups
    const int tq = (warp - 2) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_addr + tq * 128;
    const uint32_t tO = tmem + lane_addr + 256 + tq * 128;
    const int qt = my_q[tq];
    const bool mine = qt < sv.n_tiles;  // this CTA's tile of the slot exists
    const float c = a.scale_log2;
    const uint32_t pfull = lbar(L_PFULL + tq);
    float m_run = -INFINITY, l_run = 0.f;
    int cnt = 0, ncall = 0;
    bool ok = true;
    if (slot_exists(tq)) {
      TileWalk w;
      w.init(&sc, qt_last, sv.kv_n_tiles);
      int t;
      while (ok && w.next(t)) {
        if (!act(tq, t)) continue;
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_SFULL + tq), ncall & 1, wc, 321));
        if (!ok) break;
        tc_fence_after();
        const int vis = mine ? fwd::tile_vis(causal, diag, qt, t) : VIS_NONE;
        if (vis == VIS_NONE) {
          // the other CTA's rows see this key tile, these do not: P = 0
          uint32_t z[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_st16(tS + cc * 16, z);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive_cluster(pfull);
          ++ncall;
          continue;
        }
        float s[128];
        tmem_ld128(tS, s);
        if (vis == VIS_DIAG) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > r) s[i] = -INFINITY;
        } else if (t == w.n_tiles - 1) {
          const int kv_valid = ld_shared_volatile_s32(seq_smem + 16) - t * kTile;
          if (kv_valid < kTile) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= kv_valid) s[i] = -INFINITY;
          }
        }
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
        uint64_t acc[4] = {0, 0, 0, 0};
        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int e = cc * 32 + 2 * q;
            float pa, pb;
            f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), c2, nm2), pa, pb);
            pa = ex2_approx(pa);
            pb = ex2_approx(pb);
            acc[q & 3] = f2_add(acc[q & 3], f2_pack(pa, pb));
            pk[q] = pack_bf16x2(pa, pb);
          }
          tmem_st16(tS + cc * 16, pk);
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
        // the slot's previous PV finished before this S was written (one
        // thread's MMAs run in order), so O may be rescaled now
        if (ncall >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float o[32];
            tmem_ld32(tO + q4 * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + q4 * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_cluster(pfull);
        ++cnt;
        ++ncall;
      }
      // ---- epilogue (this CTA's rows of the slot)
      if (ok && ncall >= 1) ok = wait_bar(bar(B_OREADY + tq), (ncall - 1) & 1, wc, 323);
      if constexpr (kBlock) {
        ok = __all_sync(0xffffffffu, ok && mine);
      } else {
        ok = __all_sync(0xffffffffu, ok && mine && cnt >= 1);
      }
      const int tok = token_tile(sc, qt, shifted) * kTile + r;
      const bool row_in = tok < ld_shared_volatile_s32(seq_smem);
      const size_t trow =
          static_cast<size_t>(ld_shared_volatile_s32(seq_smem + 4)) + (row_in ? tok : 0);
      if (kBlock && ok) {
        tc_fence_after();
        fwd_block_epilogue(a, tO, cnt, m_run, l_run, row_in, trow, h,
                           static_cast<size_t>(ld_shared_volatile_s64(seq_smem + 8)) + tok);
      } else if (ok) {
        tc_fence_after();
        const float inv = (l_run > 0.f) ? 1.0f / l_run : 0.f;
        __nv_bfloat16* orow = a.out + (trow * a.Hq + h) * kD;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float o[32];
          __syncwarp();
          tmem_ld32(tO + q4 * 32, o);
          if (row_in) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 pk;
              pk.x = pack_bf16x2(o[v * 8 + 0] * inv, o[v * 8 + 1] * inv);
              pk.y = pack_bf16x2(o[v * 8 + 2] * inv, o[v * 8 + 3] * inv);
              pk.z = pack_bf16x2(o[v * 8 + 4] * inv, o[v * 8 + 5] * inv);
              pk.w = pack_bf16x2(o[v * 8 + 6] * inv, o[v * 8 + 7] * inv);
              *reinterpret_cast<uint4*>(orow + q4 * 32 + v * 8) = pk;
            }
          }
        }
        const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f
                                        : -INFINITY;
        if (row_in) a.lse[ld_shared_volatile_s64(seq_smem + 8) + tok] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // The leader has drained every pair MMA (bounded) before it arrives here;
  // neither CTA frees the pair's tensor memory before both are done.
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace lca
