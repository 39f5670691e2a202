// fwd_sm100.cuh -- exact attention forward, bf16, head dim 128, sm_100a.
//
// One CTA per (pair of query tiles of 128 rows, query head, batch).  Roles:
//   warp 0      TMA producer: both Q tiles once, then K and V tiles through
//               3- and 2-stage rings
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma
//   warps 2..5  softmax warpgroup of query tile 0, one row per thread
//   warps 6..9  softmax warpgroup of query tile 1
// The two warpgroups ping-pong: while one turns its S into P the tensor
// pipe runs the other tile's products, and every SM sub-partition holds two
// softmax warps to hide each other's latency.
//
// Per key/value tile j and query tile t (Ring Attention with Blockwise
// Transformers, Summary: each query block is attended block by block):
//   S_t = Q_t K_j^T                    tcgen05, bf16 x bf16 -> fp32 in TMEM
//   m   = running row max (log2 domain, scale folded in)
//   P_t = exp2(S_t*c - m) -> bf16, written back into S_t's own columns
//   O_t += P_t V_j                     tcgen05 with A = P_t read from TMEM
// with the running (m, l, O) rescaled by exp2(m_old - m_new) whenever the
// running max moves by more than 8 (log2 units).  Keeping a stale max within
// that margin is exact: numerator and denominator share it, and P stays
// below 2^8.  Moving from one key chunk to the next is the (O, lse) merge of
// the summary in unnormalised form -- the same rescale.  The MMA thread
// issues S_t for the next key tile right behind the PV that reads P_t from
// the same columns; the tensor pipe runs one thread's MMAs in order.
//
// Block calls (kBlock) attend a query block to a key/value block that
// starts elsewhere on the position axis, for a sequence-parallel ring (Ring
// Attention with Blockwise Transformers, Summary: each host keeps its query
// block, the key/value blocks travel, and the per-block results combine
// whatever their order).  The epilogue then folds this block's partial
// (O_b, lse_b) into a running float32 (O, lse) held in global memory with
// the log-sum-exp merge
//   lse = L + log(e^(lse_old - L) + e^(lse_b - L)),  L = max of the two,
//   O   = e^(lse_old - lse) O_old + e^(lse_b - lse) O_b,
// an empty partial being (0, -inf), and may also write the merged O as
// bf16.  In log2 units with this block's running (m, l): lse_b = m + log2 l
// and e^(lse_b - lse) O_b = 2^(m - lse) * (O l), the unnormalised TMEM sum.
//
// TMEM columns: S/P tile 0 [0,128) | S/P tile 1 [128,256) | O tile 0
// [256,384) | O tile 1 [384,512).
// Shared memory (1024-aligned, 128-byte swizzle): Q0 | Q1 | K x3 | V x2.
// Each 128x128 bf16 tile is two 16 KB halves (head dims 0-63, 64-127).
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "sched.cuh"

namespace lca {

namespace fwd {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr uint32_t kHalf = kTile * 64 * 2;  // 16 KB
constexpr uint32_t kTileB = 2 * kHalf;      // 32 KB
constexpr int kThreads = 320;
constexpr int kHeadBand = 4;  // heads whose CTAs are ordered together (work order)

constexpr uint32_t kOffQ = 0;                      // 2 query tiles
// Ring depths: K is read by the next S product of both query tiles right
// behind the PV that frees V, so it gets the deeper ring (225 KB of shared
// memory in all).
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kOffK = kOffQ + 2 * kTileB;             // kKStages stages
constexpr uint32_t kOffV = kOffK + kKStages * kTileB;      // kVStages stages
constexpr uint32_t kOffBar = kOffV + kVStages * kTileB;    // barriers (8 B each)
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack

// barrier indices
enum {
  B_Q = 0,
  B_KFULL = 1,                       // +stage
  B_KEMPTY = B_KFULL + kKStages,     // +stage
  B_VFULL = B_KEMPTY + kKStages,     // +stage
  B_VEMPTY = B_VFULL + kVStages,     // +stage
  B_SFULL = B_VEMPTY + kVStages,     // +query tile
  B_PFULL = B_SFULL + 2,             // +query tile, 128 arrivals
  B_OREADY = B_PFULL + 2,            // +query tile
  B_DRAIN = B_OREADY + 2,
  NUM_BARS
};
static_assert(8 * NUM_BARS + 40 <= 256, "barrier area");
// ring slot and phase of key/value tile j
__device__ __forceinline__ int kslot(int j) { return j % kKStages; }
__device__ __forceinline__ uint32_t kphase(int j) { return (j / kKStages) & 1; }
__device__ __forceinline__ int vslot(int j) { return j % kVStages; }
__device__ __forceinline__ uint32_t vphase(int j) { return (j / kVStages) & 1; }

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q K^T
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, false, true);    // P V (V MN-major)

struct Args {
  int B, Hq, Hkv;
  int S;  // tokens per batch entry of the query tensors (packed: all sequences)
  float scale_log2;
  unsigned long long budget;
  __nv_bfloat16* out;  // block calls: may be null
  float* lse;          // block calls: the running lse, read when accumulating
  float* o_acc;        // block calls: running O, [B, S, Hq, 128] float32, or null
  int accumulate;      // block calls: fold into (o_acc, lse) instead of overwriting
  AttnSched sched;
};

// Visibility of key/value position tile T to query position tile Q, whose
// diagonal key tile is Q + diag.
enum { VIS_NONE = 0, VIS_FULL = 1, VIS_DIAG = 2 };
__device__ __forceinline__ int tile_vis(bool causal, int diag, int Q, int T) {
  if (!causal) return VIS_FULL;
  const int D = Q + diag;
  return T < D ? VIS_FULL : (T == D ? VIS_DIAG : VIS_NONE);
}

// One interface over the two walks: KvWalk (chunk boundaries anywhere; each
// visit carries its key range [lo, hi)) and TileWalk (chunks of whole
// tiles; lo and hi are left alone).
__device__ __forceinline__ void walk_init(KvWalk& w, const AttnSched* s, int qt,
                                          const SeqView& v) {
  w.init(s, qt, v.kv_len);
}
__device__ __forceinline__ void walk_init(TileWalk& w, const AttnSched* s, int qt,
                                          const SeqView& v) {
  w.init(s, qt, v.kv_n_tiles);
}
__device__ __forceinline__ bool walk_next(KvWalk& w, int& t, int& lo, int& hi) {
  return w.next(t, lo, hi);
}
__device__ __forceinline__ bool walk_next(TileWalk& w, int& t, int&, int&) { return w.next(t); }

}  // namespace fwd

// Epilogue of a block call for one query row (one thread): fold this
// block's partial (TMEM O, running m and l in log2 units) into the running
// float32 (o_acc, lse) and/or write the merged row as bf16.  Every lane of
// the warp calls it (the TMEM loads are warp-collective).  Four columns at a
// time: a wider body makes the softmax loop of the block instantiation
// spill under the 168-register limit.
__device__ __forceinline__ void fwd_block_epilogue(const fwd::Args& a, uint32_t tO, int cnt,
                                                   float m_run, float l_run, bool row_in,
                                                   size_t trow, int h, size_t li) {
  using namespace fwd;
  const float L2E = 1.4426950408889634f;
  const float lb = (cnt >= 1 && l_run > 0.f) ? m_run + lg2_approx(l_run) : -INFINITY;
  const float lold = (a.accumulate && row_in) ? a.lse[li] * L2E : -INFINITY;
  const float mx = fmaxf(lb, lold);
  float ln = -INFINITY, w_old = 0.f, w_b = 0.f;
  if (mx != -INFINITY) {
    ln = mx + lg2_approx(ex2_approx(lold - mx) + ex2_approx(lb - mx));
    w_old = (lold == -INFINITY) ? 0.f : ex2_approx(lold - ln);
    w_b = (lb == -INFINITY) ? 0.f : ex2_approx(m_run - ln);
  }
  const size_t e0 = (trow * a.Hq + h) * kD;
#pragma unroll 1
  for (int q4 = 0; q4 < 4; ++q4) {
    float o[32];
    __syncwarp();
    if (cnt >= 1) {
      tmem_ld32(tO + q4 * 32, o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0.f;
    }
    if (!row_in) continue;
#pragma unroll 2
    for (int v = 0; v < 8; ++v) {
      const size_t e = e0 + q4 * 32 + 4 * v;
      float4 y = make_float4(o[4 * v] * w_b, o[4 * v + 1] * w_b, o[4 * v + 2] * w_b,
                             o[4 * v + 3] * w_b);
      if (w_old != 0.f) {
        const float4 x = *reinterpret_cast<const float4*>(a.o_acc + e);
        y.x = fmaf(w_old, x.x, y.x);
        y.y = fmaf(w_old, x.y, y.y);
        y.z = fmaf(w_old, x.z, y.z);
        y.w = fmaf(w_old, x.w, y.w);
      }
      if (a.o_acc) *reinterpret_cast<float4*>(a.o_acc + e) = y;
      if (a.out) *reinterpret_cast<uint2*>(a.out + e) = make_uint2(pack_bf16x2(y.x, y.y),
                                                                   pack_bf16x2(y.z, y.w));
    }
  }
  if (row_in) a.lse[li] = ln * 0.69314718055994531f;
}

// kRanged: some chunk boundary falls inside a tile, so visits carry key
// ranges (KvWalk).  Otherwise the cheaper tile walk runs and only a ragged
// last tile needs a key mask.  kBlock: a block call (merging epilogue).
// 320 threads: the register file is handed out in groups of four warps, so
// a CTA of ten warps is charged for twelve and may use at most 168
// registers per thread (more fails to launch).
template <bool kRanged, bool kBlock>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    attn_fwd_bf16_sm100(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ fwd::Args a) {
  using namespace fwd;
  using Walk = typename std::conditional<kRanged, KvWalk, TileWalk>::type;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * NUM_BARS + 8);
  // The sequence's length, first row, lse offset and key count, parked in
  // shared memory (re-read where needed rather than held through the
  // softmax loop): [0] len, [4] row0, [8] lse offset (64-bit), [16] kv_len
  const uint32_t seq_smem = bars + 8 * NUM_BARS + 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: a pair of query tiles.  Heads in bands of kHeadBand;
  // inside a band the longest causal pairs of all its heads come first
  // (with S2-Attn, the pairs at the same place in every group), so the grid
  // ends on short pairs, while the CTAs in flight still share a few heads'
  // K/V in L2.  (One head per band would start the last head's longest
  // pair only once the heads before it are done, and end the grid on it.)
  const AttnSched& sc = a.sched;
  const int n_pairs = (sc.n_tiles + 1) >> 1;
  const int pg_s2 = sc.s2 ? sc.group_tiles >> 1 : 0;  // pairs per S2 group
  const int pg = (pg_s2 > 0 && !(sc.group_tiles & 1) && n_pairs % pg_s2 == 0) ? pg_s2 : n_pairs;
  const int n_groups = n_pairs / pg;
  const int n_bh = a.B * a.Hq;
  const int band_cta = kHeadBand * n_pairs;
  const int band = static_cast<int>(blockIdx.x) / band_cta;
  const int in_band = static_cast<int>(blockIdx.x) - band * band_cta;
  const int band_heads = min(kHeadBand, n_bh - band * kHeadBand);
  const int slot = in_band / band_heads;  // (length class, group), longest class first
  const int pr = (slot % n_groups) * pg + (pg - 1 - slot / n_groups);
  const int bh = band * kHeadBand + in_band % band_heads;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const bool shifted = head_shifted(sc, h);
  const int qt0 = 2 * pr;
  SeqView sv;
  if (!seq_view(sc, b, a.S, &sv)) {
    if (threadIdx.x == 0 && pr == 0) record_error(kErrSeqOffsets, 150);
    return;
  }
  if (qt0 >= sv.n_tiles) return;  // a shorter packed sequence: no work here
  const bool has1 = qt0 + 1 < sv.n_tiles;
  const int qt_last = has1 ? qt0 + 1 : qt0;
  const bool causal = sc.causal != 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) {
      const uint32_t cnt = (i == B_PFULL || i == B_PFULL + 1) ? 128u : 1u;
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
      mbar_expect_tx(bar(B_Q), has1 ? 2 * kTileB : kTileB);
      for (int t = 0; t < (has1 ? 2 : 1); ++t) {
        const int tok = sv.row0 + token_tile(sc, qt0 + t, shifted) * kTile;
        tma_load_3d(sQ + t * kTileB, &tmQ, bar(B_Q), 0, h, tok);
        tma_load_3d(sQ + t * kTileB + kHalf, &tmQ, bar(B_Q), 64, h, tok);
      }
      Walk w;
      walk_init(w, &sc, qt_last, sv);
      int t, lo = 0, hi = kTile, j = 0;
      int k_issued = 0, v_issued = 0;  // tiles whose K / V copy was issued
      bool ok = true;
      while (ok && walk_next(w, t, lo, hi)) {
        const int tok = sv.kv_row0 + token_tile(sc, t, shifted) * kTile;
        const int ks = kslot(j), vs = vslot(j);
        if (j >= kKStages) ok = wait_bar(bar(B_KEMPTY + ks), kphase(j - kKStages), wc, 101);
        if (!ok) break;
        mbar_expect_tx(bar(B_KFULL + ks), kTileB);
        tma_load_3d(sK + ks * kTileB, &tmK, bar(B_KFULL + ks), 0, g, tok);
        tma_load_3d(sK + ks * kTileB + kHalf, &tmK, bar(B_KFULL + ks), 64, g, tok);
        ++k_issued;
        if (j >= kVStages) ok = wait_bar(bar(B_VEMPTY + vs), vphase(j - kVStages), wc, 102);
        if (!ok) break;
        mbar_expect_tx(bar(B_VFULL + vs), kTileB);
        tma_load_3d(sV + vs * kTileB, &tmV, bar(B_VFULL + vs), 0, g, tok);
        tma_load_3d(sV + vs * kTileB + kHalf, &tmV, bar(B_VFULL + vs), 64, g, tok);
        ++v_issued;
        ++j;
      }
      if (!ok) {
        // Unwind: let the copies already issued land before the CTA exits
        // (the last copy into each slot completes that slot's last phase).
        drain_bar(bar(B_Q), 0, 161);
        for (int x = k_issued - 1; x >= 0 && x >= k_issued - kKStages; --x)
          drain_bar(bar(B_KFULL + kslot(x)), kphase(x), 162);
        for (int x = v_issued - 1; x >= 0 && x >= v_issued - kVStages; --x)
          drain_bar(bar(B_VFULL + vslot(x)), vphase(x), 164);
      }
    }
  } else if (warp == 1) {
    // =================================================== MMA issuer
    if (lane == 0) {
      // query tiles moved onto the key tiles' diagonal (block calls)
      const int qd0 = qt0 + (kBlock ? sc.diag : 0);
      const uint32_t qts[2] = {static_cast<uint32_t>(qd0), static_cast<uint32_t>(qd0 + 1)};
      bool ok = wait_bar(bar(B_Q), 0, wc, 201);
      Walk w;
      walk_init(w, &sc, qt_last, sv);
      int T, Tn, lo = 0, hi = kTile;
      int pv_cnt[2] = {0, 0};
      // S_t for key tile j into the S/P columns of query tile t
      auto issue_s = [&](int tq, int j) {
        const uint32_t kbase = sK + kslot(j) * kTileB;
        const uint32_t qbase = sQ + tq * kTileB;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          mma_bf16_ss(tmem + tq * 128, sdesc_sw128(qbase + off, 16, 1024),
                      sdesc_sw128(kbase + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + tq));
      };
      auto act = [&](int tq, int T_) {
        return (tq == 0 || has1) && tile_vis(causal, 0, static_cast<int>(qts[tq]), T_) != VIS_NONE;
      };
      bool have = ok && walk_next(w, T, lo, hi);
      if (have) {
        ok = wait_bar(bar(B_KFULL), 0, wc, 202);
        if (ok) {
          tc_fence_after();
          if (act(0, T)) issue_s(0, 0);
          if (act(1, T)) issue_s(1, 0);
          tc_commit(bar(B_KEMPTY));
        }
      }
      int j = 0;
      while (ok && have) {
        const bool has_next = walk_next(w, Tn, lo, hi);
        ok = wait_bar(bar(B_VFULL + vslot(j)), vphase(j), wc, 203);
        if (ok && has_next) ok = wait_bar(bar(B_KFULL + kslot(j + 1)), kphase(j + 1), wc, 204);
        for (int tq = 0; tq < 2 && ok; ++tq) {
          if (act(tq, T)) {
            ok = wait_bar(bar(B_PFULL + tq), pv_cnt[tq] & 1, wc, 205);
            if (!ok) break;
            tc_fence_after();
            const uint32_t vbase = sV + vslot(j) * kTileB;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              mma_bf16_ts(tmem + 256 + tq * 128, tmem + tq * 128 + k * 8,
                          sdesc_sw128(vbase + k * 2048, kHalf, 1024), kIdescO,
                          (pv_cnt[tq] > 0 || k > 0) ? 1u : 0u);
            }
            tc_commit(bar(B_OREADY + tq));
            ++pv_cnt[tq];
          }
          if (has_next && act(tq, Tn)) issue_s(tq, j + 1);
        }
        if (!ok) break;
        tc_commit(bar(B_VEMPTY + vslot(j)));
        if (has_next) tc_commit(bar(B_KEMPTY + kslot(j + 1)));
        have = has_next;
        T = Tn;
        ++j;
      }
      // Drain: wait for every MMA this thread issued before TMEM is freed.
      tc_commit(bar(B_DRAIN));
      drain_bar(bar(B_DRAIN), 0, 166);
    }
  } else {
    // =================================================== softmax warpgroups
    const int tq = (warp - 2) >> 2;      // query tile of this warpgroup
    const int wq = warp & 3;             // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;        // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_addr + tq * 128;
    const uint32_t tO = tmem + lane_addr + 256 + tq * 128;
    // this warpgroup's query tile, moved onto the key tiles' diagonal for
    // block calls (the tile itself is recovered for the epilogue)
    const int qt_d = qt0 + tq + (kBlock ? sc.diag : 0);
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int cnt = 0;
    bool ok = true;
    if (tq == 0 || has1) {
      Walk w;
      walk_init(w, &sc, qt_last, sv);
      int t, lo = 0, hi = kTile;
      while (ok && walk_next(w, t, lo, hi)) {
        const int vis = tile_vis(causal, 0, qt_d, t);
        if (vis == VIS_NONE) continue;
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_SFULL + tq), cnt & 1, wc, 301));
        if (!ok) break;
        tc_fence_after();
        float s[128];
        tmem_ld128(tS, s);
        if constexpr (kRanged) {
          // Keys outside this visit's range [lo, hi) -- another chunk's keys
          // in a tile that straddles a chunk boundary, or rows past the end
          // of the sequence -- and, on the diagonal, keys after the row.
          const int lim = vis == VIS_DIAG ? (hi < r + 1 ? hi : r + 1) : hi;
          if (lim < kTile) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= lim) s[i] = -INFINITY;
          }
          if (lo > 0) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i < lo) s[i] = -INFINITY;
          }
        } else if (vis == VIS_DIAG) {
          // keys after the row (past the end of a ragged sequence included,
          // for every row that is stored when queries and keys are one
          // sequence; a block call's key block can end inside the diagonal
          // tile before the query rows do)
          // (a key block that ends inside a tile is one chunk of a length
          // that is not a whole number of tiles, so it takes the ranged walk,
          // which masks by key range; here every key tile is whole)
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > r) s[i] = -INFINITY;
        } else if (t == w.n_tiles - 1) {
          // last key tile of a ragged sequence: rows past its end (S2-Attn
          // sequences are whole tiles, so nothing is masked there)
          // (the key count: the sequence's length unless this is a block call)
          const int kv_valid = ld_shared_volatile_s32(seq_smem + (kBlock ? 16 : 0)) - t * kTile;
          if (kv_valid < kTile) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= kv_valid) s[i] = -INFINITY;
          }
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
        // P = 2^(s*c - m), written back as bf16 pairs over this tile's S
        // columns (16 columns per 32 keys).
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
        // The previous PV of this tile finished before this S was written
        // (one thread's MMAs run in order), so O may be rescaled now.
        if (cnt >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
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
        mbar_arrive(bar(B_PFULL + tq));
        ++cnt;
      }
      // ---- epilogue: O / l -> bf16 out, lse = ln(2) * (m + log2 l)
      if (ok && cnt >= 1) ok = wait_bar(bar(B_OREADY + tq), (cnt - 1) & 1, wc, 303);
      if constexpr (kBlock) {
        // a query tile before the key block's first diagonal sees no key: its
        // partial is empty (0, -inf) and still merges
        ok = __all_sync(0xffffffffu, ok);
      } else {
        ok = __all_sync(0xffffffffu, ok && cnt >= 1);
      }
      const int qt = qt_d - (kBlock ? sc.diag : 0);
      const int tok = token_tile(sc, qt, shifted) * kTile + r;
      // Every lane takes part in the TMEM loads (warp-collective); rows past
      // the end of the sequence (ragged last tile) only skip their stores.
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
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace lca
