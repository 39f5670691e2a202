// aux_kernels.cuh -- small memory-bound kernels around the attention passes.
//
//   bwd_rowdot   D_i = sum_c dout_ic * out_ic (float32), the row term of
//                dS = P o (dP - D) in the backward pass, plus a copy of lse,
//                both into per-sequence rows padded to whole tiles
//   dq_finalize  dq = scale * dq_acc, float32 accumulator -> bf16
//   cast_f32_bf16  float32 -> bf16 (a blockwise result's last step)
//   accumulate_f32 dst += src (ring steps' partial key/value gradients)
//   lse_merge    combine two partial (O, lse) results over disjoint key
//                sets (Ring Attention with Blockwise Transformers, Summary:
//                per-block results combine independently of order)
//   s2_roll_*    LongLoRA's shift as a row permutation, for groups whose
//                half is not a whole number of tiles
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace lca {

// One warp per padded row (sequence b, position s < S_pad, head h), h
// fastest so that neighbouring warps read neighbouring memory.  acc_zero
// (dense batches only, else null): the float32 dq accumulator, whose row
// of each visited (b, s, h) is zeroed on the way.  Sequence b
// occupies tensor rows [b*S, b*S + S) or, packed, [cu[b], cu[b+1]); lse is
// [B,H,S] or, packed, [H, total].  Writes D and a copy of lse into
// [B,H,S_pad] arrays; positions past a sequence's end get D = 0 and
// lse = +inf (P = 0 for those query rows in the backward pass).  Packed
// offsets that are out of order or out of range make the sequence empty
// here; the attention kernels report them.
template <typename T, int D>
__global__ void bwd_rowdot(const T* __restrict__ out, const T* __restrict__ dout,
                           const float* __restrict__ lse, float* __restrict__ Dst,
                           float* __restrict__ lse_pad, int B, int S, int S_pad, int H,
                           const int* __restrict__ cu_seqlens, float* __restrict__ acc_zero) {
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(B) * S_pad * H;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < n;
       w += warps) {
    int h, s, b;
    if (n <= 0xffffffffll) {  // 32-bit index arithmetic when it fits
      const uint32_t w32 = static_cast<uint32_t>(w), hs = static_cast<uint32_t>(H) * S_pad;
      h = static_cast<int>(w32 % static_cast<uint32_t>(H));
      s = static_cast<int>((w32 / static_cast<uint32_t>(H)) % static_cast<uint32_t>(S_pad));
      b = static_cast<int>(w32 / hs);
    } else {
      h = static_cast<int>(w % H);
      s = static_cast<int>((w / H) % S_pad);
      b = static_cast<int>(w / (static_cast<int64_t>(H) * S_pad));
    }
    int64_t r0 = static_cast<int64_t>(b) * S, l0 = (static_cast<int64_t>(b) * H + h) * S;
    int len = S;
    if (cu_seqlens) {
      const int c0 = cu_seqlens[b], c1 = cu_seqlens[b + 1];
      const bool valid = c0 >= 0 && c1 >= c0 && c1 <= S;
      r0 = c0;
      l0 = static_cast<int64_t>(h) * S + c0;
      len = valid ? c1 - c0 : 0;
    }
    const int64_t dst = (static_cast<int64_t>(b) * H + h) * S_pad + s;
    if (s >= len) {
      if (lane == 0) {
        Dst[dst] = 0.f;
        lse_pad[dst] = INFINITY;
      }
      continue;
    }
    const T* o = out + ((r0 + s) * H + h) * D;
    const T* g = dout + ((r0 + s) * H + h) * D;
    if (acc_zero) {
      // the row's float32 dq accumulator starts at zero (dense batches,
      // where the rows visited here are every row of the accumulator)
      float* z = acc_zero + ((r0 + s) * H + h) * D;
#pragma unroll
      for (int c = 4 * lane; c < D; c += 128)
        *reinterpret_cast<float4*>(z + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float acc = 0.f;
    if constexpr (sizeof(T) == 2 && D == 128) {
      // one 8-byte word (four bf16) of each row per lane: the warp reads
      // both 256-byte rows with one load each
      const uint2 ow = reinterpret_cast<const uint2*>(o)[lane];
      const uint2 gw = reinterpret_cast<const uint2*>(g)[lane];
      const uint32_t ov[2] = {ow.x, ow.y}, gv[2] = {gw.x, gw.y};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        // bf16 -> float: the bf16 bits are the high half of the float's
        acc = fmaf(__uint_as_float(ov[k] << 16), __uint_as_float(gv[k] << 16), acc);
        acc = fmaf(__uint_as_float(ov[k] & 0xffff0000u), __uint_as_float(gv[k] & 0xffff0000u),
                   acc);
      }
    } else {
#pragma unroll
      for (int c = lane; c < D; c += 32) {
        float ov, gv;
        if constexpr (sizeof(T) == 2) {
          ov = __bfloat162float(o[c]);
          gv = __bfloat162float(g[c]);
        } else {
          ov = o[c];
          gv = g[c];
        }
        acc = fmaf(ov, gv, acc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      Dst[dst] = acc;
      lse_pad[dst] = lse[l0 + s];
    }
  }
}

// Token held by position p of head h under LongLoRA's shift: heads from
// first_shifted on are rolled by half a group (LongLoRA, Summary).
__host__ __device__ inline int s2_token(int p, int h, int first_shifted, int half, int S) {
  return h >= first_shifted ? (p + half) % S : p;
}

// S2-Attn for groups whose half is not a whole number of tiles: shifted
// position p of a shifted head holds token (p + group/2) mod S (LongLoRA,
// Summary).  s2_roll_rows moves whole rows between the original layout
// [B, S, H, row] and the position layout (gather: position <- token;
// scatter: token <- position); heads h >= first_shifted are rolled, the
// others copied.  `vec` 16-byte words per row, one word per thread.
template <bool kScatter>
__global__ void s2_roll_rows(const uint4* __restrict__ src, uint4* __restrict__ dst, int B,
                             int S, int H, int first_shifted, int half, int vec) {
  const int64_t n = static_cast<int64_t>(B) * S * H * vec;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(i % vec);
    const int64_t row = i / vec;  // (b, p, h) in the position layout
    const int h = static_cast<int>(row % H);
    const int64_t bp = row / H;
    const int p = static_cast<int>(bp % S);
    const int64_t b = bp / S;
    const int tok = s2_token(p, h, first_shifted, half, S);
    const int64_t trow = ((b * S + tok) * H + h) * vec + w;
    if (kScatter)
      dst[trow] = src[i];
    else
      dst[i] = src[trow];
  }
}

// lse between the original layout [B, H, S] and the packed position layout
// [H, B*S] of the same roll.
template <bool kScatter>
__global__ void s2_roll_lse(const float* __restrict__ src, float* __restrict__ dst, int B, int S,
                            int H, int first_shifted, int half) {
  const int64_t n = static_cast<int64_t>(B) * S * H;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int h = static_cast<int>(i / (static_cast<int64_t>(B) * S));
    const int64_t bp = i % (static_cast<int64_t>(B) * S);  // packed position
    const int p = static_cast<int>(bp % S);
    const int64_t b = bp / S;
    const int tok = s2_token(p, h, first_shifted, half, S);
    const int64_t o = (b * H + h) * S + tok;
    if (kScatter)
      dst[o] = src[i];
    else
      dst[i] = src[o];
  }
}

// cu[i] = i * len for i = 0..n (packed offsets of n equal sequences).
__global__ void fill_offsets(int* cu, int n, int len) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x)
    cu[i] = i * len;
}

// dq(bf16) = scale * acc, 8 elements per thread.
__global__ void dq_finalize(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                            int64_t n8, float scale) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    __nv_bfloat162 r[4];
    r[0] = __floats2bfloat162_rn(a.x * scale, a.y * scale);
    r[1] = __floats2bfloat162_rn(a.z * scale, a.w * scale);
    r[2] = __floats2bfloat162_rn(b.x * scale, b.y * scale);
    r[3] = __floats2bfloat162_rn(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = *reinterpret_cast<uint4*>(r);
  }
}

// dst(bf16) = src(float32), n elements, rounded to nearest even: 8 per
// thread (both pointers 16-byte aligned), then the n % 8 tail elements.
__global__ void cast_f32_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                              int64_t n) {
  const int64_t n8 = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
    __nv_bfloat162 r[4];
    r[0] = __floats2bfloat162_rn(a.x, a.y);
    r[1] = __floats2bfloat162_rn(a.z, a.w);
    r[2] = __floats2bfloat162_rn(b.x, b.y);
    r[3] = __floats2bfloat162_rn(b.z, b.w);
    reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<uint4*>(r);
  }
  if (tid < n - n8 * 8) dst[n8 * 8 + tid] = __float2bfloat16_rn(src[n8 * 8 + tid]);
}

// dst += src, n float32 elements: 4 per thread (both pointers 16-byte
// aligned), then the n % 4 tail (a ring step's partial key/value gradients
// folded into the accumulators that travel with the block).
__global__ void accumulate_f32(const float* __restrict__ src, float* __restrict__ dst,
                               int64_t n) {
  const int64_t n4 = n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < n4; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(src)[i];
    float4 b = reinterpret_cast<float4*>(dst)[i];
    b.x += a.x;
    b.y += a.y;
    b.z += a.z;
    b.w += a.w;
    reinterpret_cast<float4*>(dst)[i] = b;
  }
  if (tid < n - n4 * 4) dst[n4 * 4 + tid] += src[n4 * 4 + tid];
}

// (O, lse) merge, one warp per row.  Every lane reads the row's two lse
// values before lane 0 overwrites lse_out, so lse_out may alias lse_a/lse_b;
// each element of o is read and written by one thread, so o_out may alias
// o_a/o_b.
__global__ void lse_merge_kernel(int64_t rows, int d, const float* o_a, const float* lse_a,
                                 const float* o_b, const float* lse_b, float* o_out,
                                 float* lse_out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += warps) {
    const float la = lse_a[r], lb = lse_b[r];
    const float M = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, l = -INFINITY;
    if (M != -INFINITY) {
      l = M + logf(expf(la - M) + expf(lb - M));
      wa = expf(la - l);
      wb = expf(lb - l);
    }
    __syncwarp();
    for (int c = lane; c < d; c += 32) {
      const int64_t i = r * d + c;
      o_out[i] = (M == -INFINITY) ? 0.f : wa * o_a[i] + wb * o_b[i];
    }
    if (lane == 0) lse_out[r] = l;
  }
}

}  // namespace lca
