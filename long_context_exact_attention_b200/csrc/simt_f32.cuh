// simt_f32.cuh -- exact attention in float32 on CUDA cores (forward and
// backward), for float32 inputs where a tensor-core path would round to
// tf32/bf16.  Tiles of 64 query rows x 64 keys, head dim 64 or 128.
//
// Forward: one CTA per (query tile, head, batch), 8 warps, each warp owning
// 8 query rows; a lane computes the logits of keys lane and lane+32 and holds
// head dims lane, lane+32, ...; row max and row sum are warp reductions
// (shuffles); the online rescale is the same (O, lse) merge as the bf16 path.
// Backward: one CTA per (key tile, key/value head, batch), looping over the
// query heads of its group and the visible query tiles; dK and dV live in
// registers, dQ is accumulated with shared-memory atomics per query tile and
// flushed to the float32 dq output with global atomics.
// Ragged and packed sequences: rows past the end of a sequence load as
// zeros and are not stored; the forward masks keys outside each visit's key
// range (which ends at the sequence's end).
#pragma once

#include "sched.cuh"

namespace lca {
namespace f32 {

constexpr int kT = 64;        // rows and keys per tile
constexpr int kThreads = 256; // 8 warps
constexpr int kRowsPerWarp = kT / (kThreads / 32);

struct Args {
  const float *q, *k, *v, *out, *lse, *dout, *D;  // lse, D: padded [B,Hq,S_pad]
  float *o_out, *lse_out, *dq, *dk, *dv;
  int B, Hq, Hkv;
  int S;      // tokens per batch entry of the tensors (packed: all sequences)
  int S_pad;  // row length of the padded lse / D copies
  float scale;
  AttnSched sched;
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_fwd_f32(const __grid_constant__ Args a) {
  constexpr int E = D / 32;      // head dims per lane
  constexpr int KP = D + 1;      // padded key row
  extern __shared__ float fsm[];
  float* sQ = fsm;               // [kT][D]
  float* sK = sQ + kT * D;       // [kT][KP]
  float* sV = sK + kT * KP;      // [kT][D]
  const AttnSched& sc = a.sched;
  const int BH = a.B * a.Hq;
  const int qt = sc.n_tiles - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int h = bh % a.Hq, b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  SeqView sv;
  if (!seq_view(sc, b, a.S, &sv)) {
    if (threadIdx.x == 0 && qt == 0) record_error(kErrSeqOffsets, 160);
    return;
  }
  if (qt >= sv.n_tiles) return;  // a shorter packed sequence: no work here
  const size_t row0 = static_cast<size_t>(sv.bm) * a.S + sv.tokb;  // first row of the sequence
  const bool shifted = head_shifted(sc, h);
  const int qtok0 = token_tile(sc, qt, shifted) * kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < kT * D; i += kThreads) {
    const int r = i / D, c = i % D;
    sQ[i] = (qtok0 + r < sv.len) ? a.q[((row0 + qtok0 + r) * a.Hq + h) * D + c] : 0.f;
  }
  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][E];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[rr][e] = 0.f;
  }
  KvWalk w;
  w.init(&sc, qt, sv.len);
  int t, lo, hi;
  while (w.next(t, lo, hi)) {
    const int ktok0 = token_tile(sc, t, shifted) * kT;
    __syncthreads();
    for (int i = threadIdx.x; i < kT * D; i += kThreads) {
      const int r = i / D, c = i % D;
      const bool in = ktok0 + r < sv.len;
      const size_t src = ((row0 + (in ? ktok0 + r : 0)) * a.Hkv + g) * D + c;
      sK[r * KP + c] = in ? a.k[src] : 0.f;
      sV[r * D + c] = in ? a.v[src] : 0.f;
    }
    __syncthreads();
    const bool diag = sc.causal && t == qt;
#pragma unroll 1
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = warp * kRowsPerWarp + rr;
      float s0 = 0.f, s1 = 0.f;
      for (int c = 0; c < D; ++c) {
        const float qv = sQ[r * D + c];
        s0 = fmaf(qv, sK[lane * KP + c], s0);
        s1 = fmaf(qv, sK[(lane + 32) * KP + c], s1);
      }
      s0 *= a.scale;
      s1 *= a.scale;
      // keys outside this visit's range [lo, hi), and after the row on the diagonal
      if ((diag && lane > r) || lane < lo || lane >= hi) s0 = -INFINITY;
      if ((diag && lane + 32 > r) || lane + 32 < lo || lane + 32 >= hi) s1 = -INFINITY;
      const float mx = warp_max(fmaxf(s0, s1));
      const float m_new = fmaxf(m[rr], mx);
      const float alpha = (m[rr] == -INFINITY) ? 0.f : expf(m[rr] - m_new);
      const float p0 = expf(s0 - m_new), p1 = expf(s1 - m_new);
      l[rr] = l[rr] * alpha + warp_sum(p0 + p1);
      m[rr] = m_new;
#pragma unroll
      for (int e = 0; e < E; ++e) o[rr][e] *= alpha;
      for (int j = 0; j < 32; ++j) {
        const float pa = __shfl_sync(0xffffffffu, p0, j);
        const float pb = __shfl_sync(0xffffffffu, p1, j);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          o[rr][e] = fmaf(pa, sV[j * D + lane + 32 * e], o[rr][e]);
          o[rr][e] = fmaf(pb, sV[(j + 32) * D + lane + 32 * e], o[rr][e]);
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int r = warp * kRowsPerWarp + rr;
    const int tok = qtok0 + r;
    if (tok >= sv.len) continue;
    const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
    float* orow = a.o_out + ((row0 + tok) * a.Hq + h) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) orow[lane + 32 * e] = o[rr][e] * inv;
    if (lane == 0)
      a.lse_out[(static_cast<size_t>(sv.bm) * a.Hq + h) * a.S + sv.tokb + tok] =
          l[rr] > 0.f ? m[rr] + logf(l[rr]) : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_bwd_f32(const __grid_constant__ Args a) {
  constexpr int E = D / 32;
  constexpr int P = D + 1;
  extern __shared__ float fsm[];
  float* sK = fsm;               // [kT][D]
  float* sV = sK + kT * D;       // [kT][D]
  float* sQ = sV + kT * D;       // [kT][P]
  float* sO = sQ + kT * P;       // dO [kT][P]
  float* sdQ = sO + kT * P;      // [kT][D]
  float* sL = sdQ + kT * D;      // lse [kT]
  float* sD = sL + kT;           // D [kT]
  const AttnSched& sc = a.sched;
  const int rep = a.Hq / a.Hkv;
  const int BG = a.B * a.Hkv;
  const int kt = static_cast<int>(blockIdx.x) / BG;
  const int bg = static_cast<int>(blockIdx.x) % BG;
  const int g = bg % a.Hkv, b = bg / a.Hkv;
  SeqView sv;
  if (!seq_view(sc, b, a.S, &sv)) {
    if (threadIdx.x == 0 && kt == 0) record_error(kErrSeqOffsets, 161);
    return;
  }
  if (kt >= sv.n_tiles) return;  // a shorter packed sequence: no work here
  const size_t row0 = static_cast<size_t>(sv.bm) * a.S + sv.tokb;
  const bool shifted = head_shifted(sc, g * rep);
  const int ktok0 = token_tile(sc, kt, shifted) * kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < kT * D; i += kThreads) {
    const int r = i / D, c = i % D;
    const bool in = ktok0 + r < sv.len;
    const size_t src = ((row0 + (in ? ktok0 + r : 0)) * a.Hkv + g) * D + c;
    sK[i] = in ? a.k[src] : 0.f;
    sV[i] = in ? a.v[src] : 0.f;
  }
  float dk[kRowsPerWarp][E], dv[kRowsPerWarp][E];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
    for (int e = 0; e < E; ++e) dk[rr][e] = dv[rr][e] = 0.f;

  QWalk qw;
  qw.init(&sc, kt, sv.n_tiles);
  for (int hr = 0; hr < rep; ++hr) {
    const int h = g * rep + hr;
    for (int qt = qw.t; qt < qw.t_end; ++qt) {
      const int qtok0 = token_tile(sc, qt, shifted) * kT;
      __syncthreads();
      for (int i = threadIdx.x; i < kT * D; i += kThreads) {
        const int r = i / D, c = i % D;
        const bool in = qtok0 + r < sv.len;
        const size_t src = ((row0 + (in ? qtok0 + r : 0)) * a.Hq + h) * D + c;
        sQ[r * P + c] = in ? a.q[src] : 0.f;
        sO[r * P + c] = in ? a.dout[src] : 0.f;
        sdQ[i] = 0.f;
      }
      for (int i = threadIdx.x; i < kT; i += kThreads) {
        const size_t ri = (static_cast<size_t>(b) * a.Hq + h) * a.S_pad + qtok0 + i;
        sL[i] = a.lse[ri];
        sD[i] = a.D[ri];
      }
      __syncthreads();
      const bool diag = sc.causal && qt == kt;
#pragma unroll 1
      for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int j = warp * kRowsPerWarp + rr;   // key row
        float s0 = 0.f, s1 = 0.f, dp0 = 0.f, dp1 = 0.f;
        for (int c = 0; c < D; ++c) {
          const float kv = sK[j * D + c], vv = sV[j * D + c];
          s0 = fmaf(sQ[lane * P + c], kv, s0);
          s1 = fmaf(sQ[(lane + 32) * P + c], kv, s1);
          dp0 = fmaf(sO[lane * P + c], vv, dp0);
          dp1 = fmaf(sO[(lane + 32) * P + c], vv, dp1);
        }
        float p0 = expf(s0 * a.scale - sL[lane]);
        float p1 = expf(s1 * a.scale - sL[lane + 32]);
        if (diag && j > lane) p0 = 0.f;
        if (diag && j > lane + 32) p1 = 0.f;
        const float ds0 = p0 * (dp0 - sD[lane]);
        const float ds1 = p1 * (dp1 - sD[lane + 32]);
        for (int i = 0; i < 32; ++i) {
          const float pa = __shfl_sync(0xffffffffu, p0, i);
          const float pb = __shfl_sync(0xffffffffu, p1, i);
          const float da = __shfl_sync(0xffffffffu, ds0, i);
          const float db = __shfl_sync(0xffffffffu, ds1, i);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int c = lane + 32 * e;
            dv[rr][e] = fmaf(pa, sO[i * P + c], dv[rr][e]);
            dv[rr][e] = fmaf(pb, sO[(i + 32) * P + c], dv[rr][e]);
            dk[rr][e] = fmaf(da, sQ[i * P + c], dk[rr][e]);
            dk[rr][e] = fmaf(db, sQ[(i + 32) * P + c], dk[rr][e]);
          }
        }
        // dQ_i += scale * dS_ij k_j  (rows lane, lane+32)
        for (int c = 0; c < D; ++c) {
          const float kv = sK[j * D + c] * a.scale;
          atomicAdd(&sdQ[lane * D + c], ds0 * kv);
          atomicAdd(&sdQ[(lane + 32) * D + c], ds1 * kv);
        }
      }
      __syncthreads();
      for (int i = threadIdx.x; i < kT * D; i += kThreads) {
        const int r = i / D, c = i % D;
        if (qtok0 + r < sv.len) atomicAdd(&a.dq[((row0 + qtok0 + r) * a.Hq + h) * D + c], sdQ[i]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int j = warp * kRowsPerWarp + rr;
    if (ktok0 + j >= sv.len) continue;
    const size_t dst = ((row0 + ktok0 + j) * a.Hkv + g) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      a.dk[dst + lane + 32 * e] = dk[rr][e] * a.scale;
      a.dv[dst + lane + 32 * e] = dv[rr][e];
    }
  }
}

template <int D>
constexpr size_t fwd_smem() { return sizeof(float) * (kT * D + kT * (D + 1) + kT * D); }
template <int D>
constexpr size_t bwd_smem() {
  return sizeof(float) * (2 * kT * D + 2 * kT * (D + 1) + kT * D + 2 * kT);
}

}  // namespace f32
}  // namespace lca
