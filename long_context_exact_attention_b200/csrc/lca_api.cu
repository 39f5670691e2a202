// lca_api.cu -- the C ABI of liblca (declared in include/lca.h): argument
// validation, TMA descriptor encoding, launch configuration.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/lca.h"
#include "aux_kernels.cuh"
#include "bwd_sm100.cuh"
#include "ffn_sm100.cuh"
#include "fwd_sm100.cuh"
#include "ptx.cuh"
#include "sched.cuh"
#include "simt_f32.cuh"

using namespace lca;

namespace {

thread_local std::string t_last_error = "no error";

lca_status fail(lca_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = std::string(lca_status_string(s)) + ": " + buf;
  return s;
}

lca_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LCA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr unsigned long long kDefaultBudget = 1ull << 31;

struct Common {
  int B, Hq, Hkv, S, d;  // tensor extents: B batch entries of S tokens (packed: 1 x total)
  int S_kv;              // key/value tokens per batch entry (block calls; else S)
  int n_seq;             // sequences (B unless packed)
  int S_seq;             // longest sequence (S unless packed)
  const int* cu;         // packed token offsets (device), else null
  int dtype;
  float scale;
  int tile;
};

// The longest sequence rounded up to the tile of the element type's path.
int s_pad_of(const Common& c) { return (c.S_seq + c.tile - 1) / c.tile * c.tile; }

lca_status check_shape(const lca_shape* sh, Common* c) {
  if (!sh) return fail(LCA_ERR_INVALID_ARG, "shape is NULL");
  if (sh->B <= 0 || sh->Hq <= 0 || sh->Hkv <= 0 || sh->S <= 0 || sh->d <= 0)
    return fail(LCA_ERR_INVALID_ARG, "dimensions must be positive");
  if (sh->Hq % sh->Hkv) return fail(LCA_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (sh->B > (1 << 20) || sh->Hq > 4096 || sh->S > (1ll << 26))
    return fail(LCA_ERR_INVALID_ARG, "dimension too large");
  if (sh->B * sh->S > (1ll << 31) - 1)
    return fail(LCA_ERR_INVALID_ARG, "B*S must fit in 31 bits");
  if (sh->dtype != LCA_BF16 && sh->dtype != LCA_FP32)
    return fail(LCA_ERR_INVALID_ARG, "unknown dtype %d", sh->dtype);
  if (!(sh->scale >= 0.f) || std::isinf(sh->scale))
    return fail(LCA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  c->B = static_cast<int>(sh->B);
  c->Hq = static_cast<int>(sh->Hq);
  c->Hkv = static_cast<int>(sh->Hkv);
  c->S = static_cast<int>(sh->S);
  c->S_kv = c->S;
  c->d = static_cast<int>(sh->d);
  c->n_seq = c->B;
  c->S_seq = c->S;
  c->cu = nullptr;
  c->dtype = sh->dtype;
  c->scale = sh->scale > 0.f ? sh->scale : 1.0f / std::sqrt(static_cast<float>(sh->d));
  if (sh->dtype == LCA_BF16) {
    if (sh->d != 128) return fail(LCA_ERR_UNSUPPORTED, "bf16 path needs d == 128 (got %lld)",
                                  static_cast<long long>(sh->d));
    c->tile = 128;
  } else {
    if (sh->d != 64 && sh->d != 128)
      return fail(LCA_ERR_UNSUPPORTED, "fp32 path needs d in {64, 128}");
    c->tile = 64;
  }
  return LCA_OK;
}

// Packed variable-length batch: shape->B sequences whose tokens are
// concatenated along one axis of shape->S tokens, sequence b holding tokens
// [cu_seqlens[b], cu_seqlens[b+1]), none longer than max_seqlen.
lca_status check_packed(const lca_shape* sh, const int32_t* cu_seqlens, int64_t max_seqlen,
                        Common* c) {
  if (!sh) return fail(LCA_ERR_INVALID_ARG, "shape is NULL");
  // the tensors hold one batch entry of S = total tokens; B counts sequences
  lca_shape one = *sh;
  one.B = 1;
  lca_status r = check_shape(&one, c);
  if (r != LCA_OK) return r;
  if (sh->B <= 0 || sh->B > (1 << 20))
    return fail(LCA_ERR_INVALID_ARG, "sequence count must lie in [1, 2^20]");
  c->B = static_cast<int>(sh->B);
  if (!cu_seqlens) return fail(LCA_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)
    return fail(LCA_ERR_INVALID_ARG, "cu_seqlens not 4-byte aligned");
  if (max_seqlen <= 0 || max_seqlen > sh->S)
    return fail(LCA_ERR_INVALID_ARG, "max_seqlen must lie in [1, total tokens]");
  c->n_seq = c->B;
  c->B = 1;
  c->S_seq = static_cast<int>(max_seqlen);
  c->cu = cu_seqlens;
  return LCA_OK;
}

lca_status check_ptrs(std::initializer_list<const void*> ps) {
  int i = 0;
  for (const void* p : ps) {
    if (!p) return fail(LCA_ERR_INVALID_ARG, "pointer argument %d is NULL", i);
    if (!aligned16(p)) return fail(LCA_ERR_INVALID_ARG, "pointer argument %d not 16-byte aligned", i);
    ++i;
  }
  return LCA_OK;
}

// Chunked (ring-simulating) schedule.
lca_status make_chunk_sched(const Common& c, int causal, int64_t kv_chunk, const lca_opts* o,
                            AttnSched* s) {
  std::memset(s, 0, sizeof *s);
  s->S = c.S_seq;
  s->tile = c.tile;
  s->n_tiles = (c.S_seq + c.tile - 1) / c.tile;
  s->S_kv = s->S;
  s->n_kv_tiles = s->n_tiles;
  s->causal = causal ? 1 : 0;
  s->cu_seqlens = c.cu;
  if (kv_chunk < 0) return fail(LCA_ERR_INVALID_ARG, "kv_chunk must be >= 0");
  const int64_t chunk = kv_chunk == 0 || kv_chunk > c.S_seq ? c.S_seq : kv_chunk;
  s->kv_chunk = static_cast<int>(chunk);
  const int64_t n_chunks = (c.S_seq + chunk - 1) / chunk;
  if (n_chunks > LCA_MAX_CHUNKS)
    return fail(LCA_ERR_INVALID_ARG, "%lld chunks exceed LCA_MAX_CHUNKS",
                static_cast<long long>(n_chunks));
  s->n_chunks = static_cast<int>(n_chunks);
  s->order = o ? o->order : LCA_ORDER_INORDER;
  if (s->order < 0 || s->order > 2) return fail(LCA_ERR_INVALID_ARG, "unknown chunk order");
  const int64_t qb = (o && o->q_block) ? o->q_block : chunk;
  if (qb <= 0) return fail(LCA_ERR_INVALID_ARG, "q_block must be positive");
  s->q_block = static_cast<int>(qb > c.S_seq ? c.S_seq : qb);
  if (s->order == LCA_ORDER_CUSTOM && c.cu)
    return fail(LCA_ERR_INVALID_ARG,
                "CUSTOM chunk order needs one chunk count; packed sequences have several");
  if (s->order == LCA_ORDER_CUSTOM) {
    if (!o->chunk_perm) return fail(LCA_ERR_INVALID_ARG, "CUSTOM order needs chunk_perm");
    bool seen[LCA_MAX_CHUNKS] = {};
    for (int i = 0; i < s->n_chunks; ++i) {
      const int v = o->chunk_perm[i];
      if (v < 0 || v >= s->n_chunks || seen[v])
        return fail(LCA_ERR_INVALID_ARG, "chunk_perm is not a permutation of 0..%d",
                    s->n_chunks - 1);
      seen[v] = true;
      s->perm[i] = static_cast<uint16_t>(v);
    }
  }
  return LCA_OK;
}

lca_status make_s2_sched(const Common& c, int causal, int64_t group, int64_t shift_heads,
                         AttnSched* s) {
  std::memset(s, 0, sizeof *s);
  if (group <= 0 || c.S % group || group % 2 || (group / 2) % c.tile)
    return fail(LCA_ERR_INVALID_ARG,
                "group must divide S and group/2 must be a multiple of %d", c.tile);
  if (shift_heads < 0 || shift_heads > c.Hq)
    return fail(LCA_ERR_INVALID_ARG, "shift_heads outside [0, Hq]");
  const int rep = c.Hq / c.Hkv;
  if ((c.Hq - shift_heads) % rep)
    return fail(LCA_ERR_INVALID_ARG, "shifted heads must cover whole grouped-query groups");
  s->S = c.S;
  s->tile = c.tile;
  s->n_tiles = c.S / c.tile;
  s->S_kv = s->S;
  s->n_kv_tiles = s->n_tiles;
  s->causal = causal ? 1 : 0;
  s->s2 = 1;
  s->n_chunks = 1;
  s->kv_chunk = c.S;
  s->q_block = c.S;
  s->group_tiles = static_cast<int>(group / c.tile);
  s->shift_tiles = static_cast<int>(group / 2 / c.tile);
  s->first_shifted_head = static_cast<int>(c.Hq - shift_heads);
  return LCA_OK;
}

// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B][S][heads][128] bf16 viewed 3-D (head dim, head, token on the flattened
// axis of all B*S rows); box = 64 head dims x 1 head x 128 tokens.  Rows
// past the last token load as zeros; a ragged tile otherwise reads the
// following batch entry's rows, which the kernels mask.
lca_status make_map(CUtensorMap* m, const void* ptr, int64_t B, int64_t S, int64_t heads) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(B * S)};
  const cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(heads) * 128 * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LCA_OK;
}

// fp32 [B][S][heads][128] accumulator viewed 3-D like make_map; box = 32
// head dims x 1 head x 64 tokens, no swizzle (the box's rows are 128 bytes);
// reduce-adds of rows past the last token are dropped.
lca_status make_map_acc(CUtensorMap* m, const void* ptr, int64_t B, int64_t S, int64_t heads) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(B * S)};
  const cuuint64_t strides[2] = {128 * 4, static_cast<cuuint64_t>(heads) * 128 * 4};
  const cuuint32_t box[3] = {32, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LCA_OK;
}

// [rows][cols] bf16 row-major viewed 2-D; box = 64 columns x box_rows rows,
// 128-byte swizzle: 128 rows for a K-major operand tile of the feedforward
// products, 64 rows for an MN-major one.  Rows past the extent load as zeros.
lca_status make_map_2d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols,
                       uint32_t box_rows = 128, int64_t row_stride = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride ? row_stride : cols) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LCA_OK;
}

// Streaming multiprocessors of the current device (cached per device).
lca_status sm_count(int* n) {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64 && cache[dev]) {
    *n = cache[dev];
    return LCA_OK;
  }
  int v = 0;
  e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
  if (dev >= 0 && dev < 64) cache[dev] = v;
  *n = v;
  return LCA_OK;
}

// The backward kernel's warpgroups redistribute registers with setmaxnreg;
// the split adds up to exactly the registers the CTA is launched with, so
// refuse to launch a build whose register count differs.
template <bool kAccKV>
lca_status check_bwd_regs() {
  static int regs = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (regs < 0) {
    cudaFuncAttributes attr{};
    const cudaError_t e = cudaFuncGetAttributes(&attr, attn_bwd_bf16_sm100<kAccKV>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(backward)");
    regs = attr.numRegs;
  }
  if (regs != bwd::kRegsLaunch)
    return fail(LCA_ERR_UNSUPPORTED,
                "backward kernel built with %d registers per thread; its register split "
                "needs exactly %d",
                regs, bwd::kRegsLaunch);
  return LCA_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device; `slot`
// names the kernel (one per instantiation, below kSmemSlots).
constexpr int kSmemSlots = 24;
template <typename K>
lca_status ensure_smem(K kernel, size_t bytes, int slot) {
  static std::mutex mu;
  static bool done[64][kSmemSlots] = {};
  if (slot < 0 || slot >= kSmemSlots) return fail(LCA_ERR_CUDA, "internal: bad kernel slot");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 64 && done[dev][slot]) return LCA_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  if (dev < 64) done[dev][slot] = true;
  return LCA_OK;
}

lca_status launched(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return LCA_OK;
}

unsigned long long budget_of(const lca_opts* o) {
  return (o && o->timeout_cycles) ? o->timeout_cycles : kDefaultBudget;
}

// ---------------------------------------------------------------- forward
// Block calls pass o_acc (may be null when out is given) and `accumulate`;
// `block` selects the merging epilogue.
struct FwdBlock {
  bool block = false;
  float* o_acc = nullptr;
  int accumulate = 0;
};

lca_status run_fwd(const Common& c, const AttnSched& s, const void* q, const void* k,
                   const void* v, void* out, float* lse, unsigned long long budget,
                   cudaStream_t st, const FwdBlock& fb = FwdBlock()) {
  const int64_t grid64 = static_cast<int64_t>(s.n_tiles) * c.n_seq * c.Hq;
  if (grid64 > 0x7fffffffll)
    return fail(LCA_ERR_INVALID_ARG, "%lld query tiles exceed one launch",
                static_cast<long long>(grid64));
  const unsigned grid = static_cast<unsigned>(grid64);
  if (c.dtype == LCA_BF16) {
    // one CTA per pair of 128-row query tiles
    const unsigned grid2 = static_cast<unsigned>((s.n_tiles + 1) / 2) * c.n_seq * c.Hq;
    CUtensorMap mq, mk, mv;
    lca_status r;
    if ((r = make_map(&mq, q, c.B, c.S, c.Hq)) != LCA_OK) return r;
    if ((r = make_map(&mk, k, c.B, c.S_kv, c.Hkv)) != LCA_OK) return r;
    if ((r = make_map(&mv, v, c.B, c.S_kv, c.Hkv)) != LCA_OK) return r;
    // chunk boundaries inside a tile need the ranged walk
    const bool ranged = !s.s2 && s.kv_chunk % c.tile != 0;
    if (fb.block) {
      if (ranged) {
        if ((r = ensure_smem(attn_fwd_bf16_sm100<true, true>, fwd::kSmemBytes, 14)) != LCA_OK)
          return r;
      } else {
        if ((r = ensure_smem(attn_fwd_bf16_sm100<false, true>, fwd::kSmemBytes, 13)) != LCA_OK)
          return r;
      }
    } else if (ranged) {
      if ((r = ensure_smem(attn_fwd_bf16_sm100<true, false>, fwd::kSmemBytes, 6)) != LCA_OK)
        return r;
    } else {
      if ((r = ensure_smem(attn_fwd_bf16_sm100<false, false>, fwd::kSmemBytes, 0)) != LCA_OK)
        return r;
    }
    fwd::Args a;
    a.B = c.n_seq;
    a.Hq = c.Hq;
    a.Hkv = c.Hkv;
    a.S = c.S;
    a.scale_log2 = c.scale * 1.4426950408889634f;
    a.budget = budget;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.o_acc = fb.o_acc;
    a.accumulate = fb.accumulate;
    a.sched = s;
    if (fb.block && ranged)
      attn_fwd_bf16_sm100<true, true><<<grid2, fwd::kThreads, fwd::kSmemBytes, st>>>(mq, mk, mv,
                                                                                      a);
    else if (fb.block)
      attn_fwd_bf16_sm100<false, true><<<grid2, fwd::kThreads, fwd::kSmemBytes, st>>>(mq, mk, mv,
                                                                                       a);
    else if (ranged)
      attn_fwd_bf16_sm100<true, false><<<grid2, fwd::kThreads, fwd::kSmemBytes, st>>>(mq, mk, mv,
                                                                                       a);
    else
      attn_fwd_bf16_sm100<false, false><<<grid2, fwd::kThreads, fwd::kSmemBytes, st>>>(mq, mk,
                                                                                        mv, a);
    return launched("attn_fwd_bf16_sm100");
  }
  f32::Args a{};
  a.q = static_cast<const float*>(q);
  a.k = static_cast<const float*>(k);
  a.v = static_cast<const float*>(v);
  a.o_out = static_cast<float*>(out);
  a.lse_out = lse;
  a.B = c.n_seq;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.S = c.S;
  a.S_pad = s_pad_of(c);
  a.scale = c.scale;
  a.sched = s;
  lca_status r;
  if (c.d == 64) {
    if ((r = ensure_smem(f32::attn_fwd_f32<64>, f32::fwd_smem<64>(), 1)) != LCA_OK) return r;
    f32::attn_fwd_f32<64><<<grid, f32::kThreads, f32::fwd_smem<64>(), st>>>(a);
  } else {
    if ((r = ensure_smem(f32::attn_fwd_f32<128>, f32::fwd_smem<128>(), 2)) != LCA_OK) return r;
    f32::attn_fwd_f32<128><<<grid, f32::kThreads, f32::fwd_smem<128>(), st>>>(a);
  }
  return launched("attn_fwd_f32");
}

// ---------------------------------------------------------------- backward
// Workspace: D rows and a copy of lse, each [n_seq][Hq][S_pad] with S_pad
// the longest sequence rounded up to the tile, then (bf16) the fp32 dq
// accumulator over every token row.
size_t ws_d_bytes(const Common& c) {
  const size_t n = static_cast<size_t>(c.n_seq) * c.Hq * s_pad_of(c) * sizeof(float);
  return (n + 255) & ~static_cast<size_t>(255);
}
size_t ws_bytes_of(const Common& c) {
  size_t n = 2 * ws_d_bytes(c);
  if (c.dtype == LCA_BF16) n += static_cast<size_t>(c.B) * c.S * c.Hq * c.d * sizeof(float);
  return n;
}

// bf16 backward in three phases over the workspace (D | lse copy | dq
// accumulator): prep (zero the accumulator, D rows and the padded lse copy),
// main (the tensor-core kernel: dK/dV of every key tile, dQ added into the
// accumulator), dq (scale and round the accumulator).  lca_attn_bwd runs
// all three; block calls run prep once per query block, main once per key
// block, and dq at the end.
lca_status bwd_prep(const Common& c, const void* out, const float* lse, const void* dout,
                    void* ws, cudaStream_t st) {
  const int S_pad = s_pad_of(c);
  float* Drow = static_cast<float*>(ws);
  float* lse_pad = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_d_bytes(c));
  float* acc = reinterpret_cast<float*>(static_cast<char*>(ws) + 2 * ws_d_bytes(c));
  const int64_t rows = static_cast<int64_t>(c.B) * c.S * c.Hq;
  const int64_t pad_rows = static_cast<int64_t>(c.n_seq) * S_pad * c.Hq;
  const unsigned rd_blocks =
      static_cast<unsigned>(std::min<int64_t>((pad_rows * 32 + 255) / 256, 148 * 64));
  // A dense batch: the row-dot visits every row of the accumulator and
  // zeroes it on the way; a packed one may leave rows between sequences.
  if (c.cu) {
    const cudaError_t e =
        cudaMemsetAsync(acc, 0, static_cast<size_t>(rows) * c.d * sizeof(float), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dq accumulator)");
  }
  bwd_rowdot<__nv_bfloat16, 128><<<rd_blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, Drow,
      lse_pad, c.n_seq, c.S, S_pad, c.Hq, c.cu, c.cu ? nullptr : acc);
  return launched("bwd_rowdot");
}

// dk/dv (bf16, overwritten) or dk_acc/dv_acc (float32, added to when
// acc_add, else overwritten): exactly one pair is non-null.
lca_status bwd_main(const Common& c, const AttnSched& s, const void* q, const void* k,
                    const void* v, const void* dout, void* ws, void* dk, void* dv, float* dk_acc,
                    float* dv_acc, int acc_add, unsigned long long budget, cudaStream_t st) {
  const int S_pad = s_pad_of(c);
  float* Drow = static_cast<float*>(ws);
  float* lse_pad = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_d_bytes(c));
  float* acc = reinterpret_cast<float*>(static_cast<char*>(ws) + 2 * ws_d_bytes(c));
  const int64_t grid64 = static_cast<int64_t>(s.n_kv_tiles) * c.n_seq * c.Hkv;
  if (grid64 > 0x7fffffffll)
    return fail(LCA_ERR_INVALID_ARG, "%lld key tiles exceed one launch",
                static_cast<long long>(grid64));
  const unsigned grid = static_cast<unsigned>(grid64);
  const bool acc_kv = dk_acc != nullptr;
  lca_status r;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if ((r = make_map(&mq, q, c.B, c.S, c.Hq)) != LCA_OK) return r;
  if ((r = make_map(&mk, k, c.B, c.S_kv, c.Hkv)) != LCA_OK) return r;
  if ((r = make_map(&mv, v, c.B, c.S_kv, c.Hkv)) != LCA_OK) return r;
  if ((r = make_map(&mdo, dout, c.B, c.S, c.Hq)) != LCA_OK) return r;
  if ((r = make_map_acc(&mdq, acc, c.B, c.S, c.Hq)) != LCA_OK) return r;
  if (acc_kv) {
    if ((r = check_bwd_regs<true>()) != LCA_OK) return r;
    if ((r = ensure_smem(attn_bwd_bf16_sm100<true>, bwd::kSmemBytes, 15)) != LCA_OK) return r;
  } else {
    if ((r = check_bwd_regs<false>()) != LCA_OK) return r;
    if ((r = ensure_smem(attn_bwd_bf16_sm100<false>, bwd::kSmemBytes, 3)) != LCA_OK) return r;
  }
  bwd::Args a;
  a.B = c.n_seq;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.S = c.S;
  a.S_pad = S_pad;
  a.scale = c.scale;
  a.scale_log2 = c.scale * 1.4426950408889634f;
  a.budget = budget;
  a.lse = lse_pad;
  a.Drow = Drow;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dk_acc = dk_acc;
  a.dv_acc = dv_acc;
  a.acc_add = acc_add;
  a.sched = s;
  if (acc_kv)
    attn_bwd_bf16_sm100<true><<<grid, bwd::kThreads, bwd::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq,
                                                                            a);
  else
    attn_bwd_bf16_sm100<false><<<grid, bwd::kThreads, bwd::kSmemBytes, st>>>(mq, mk, mv, mdo,
                                                                             mdq, a);
  return launched("attn_bwd_bf16_sm100");
}

lca_status bwd_dq(const Common& c, const void* ws, void* dq, cudaStream_t st) {
  const float* acc =
      reinterpret_cast<const float*>(static_cast<const char*>(ws) + 2 * ws_d_bytes(c));
  const int64_t n8 = static_cast<int64_t>(c.B) * c.S * c.Hq * c.d / 8;
  dq_finalize<<<static_cast<unsigned>(std::min<int64_t>((n8 + 255) / 256, 148 * 16)), 256, 0,
                st>>>(acc, static_cast<__nv_bfloat16*>(dq), n8, c.scale);
  return launched("dq_finalize");
}

lca_status check_ws(const Common& c, const void* ws, size_t ws_bytes) {
  if (!ws) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  if (ws_bytes < ws_bytes_of(c))
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes,
                ws_bytes_of(c));
  if (!aligned16(ws)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  return LCA_OK;
}

lca_status run_bwd(const Common& c, const AttnSched& s, const void* q, const void* k,
                   const void* v, const void* out, const float* lse, const void* dout, void* dq,
                   void* dk, void* dv, void* ws, size_t ws_bytes, unsigned long long budget,
                   cudaStream_t st) {
  lca_status r = check_ws(c, ws, ws_bytes);
  if (r != LCA_OK) return r;
  const int S_pad = s_pad_of(c);
  float* Drow = static_cast<float*>(ws);
  float* lse_pad = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_d_bytes(c));
  const int64_t rows = static_cast<int64_t>(c.B) * c.S * c.Hq;
  const int64_t pad_rows = static_cast<int64_t>(c.n_seq) * S_pad * c.Hq;
  const unsigned rd_blocks =
      static_cast<unsigned>(std::min<int64_t>((pad_rows * 32 + 255) / 256, 148 * 64));
  const int64_t grid64 = static_cast<int64_t>(s.n_tiles) * c.n_seq * c.Hkv;
  if (grid64 > 0x7fffffffll)
    return fail(LCA_ERR_INVALID_ARG, "%lld key tiles exceed one launch",
                static_cast<long long>(grid64));
  const unsigned grid = static_cast<unsigned>(grid64);
  cudaError_t e;
  if (c.dtype == LCA_BF16) {
    if ((r = bwd_prep(c, out, lse, dout, ws, st)) != LCA_OK) return r;
    if ((r = bwd_main(c, s, q, k, v, dout, ws, dk, dv, nullptr, nullptr, 0, budget, st)) !=
        LCA_OK)
      return r;
    return bwd_dq(c, ws, dq, st);
  }
  // fp32
  e = cudaMemsetAsync(dq, 0, static_cast<size_t>(rows) * c.d * sizeof(float), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dq)");
  if (c.d == 64)
    bwd_rowdot<float, 64><<<rd_blocks, 256, 0, st>>>(static_cast<const float*>(out),
                                                       static_cast<const float*>(dout), lse, Drow,
                                                       lse_pad, c.n_seq, c.S, S_pad, c.Hq, c.cu,
                                                       nullptr);
  else
    bwd_rowdot<float, 128><<<rd_blocks, 256, 0, st>>>(static_cast<const float*>(out),
                                                        static_cast<const float*>(dout), lse,
                                                        Drow, lse_pad, c.n_seq, c.S, S_pad, c.Hq,
                                                        c.cu, nullptr);
  if ((r = launched("bwd_rowdot")) != LCA_OK) return r;
  f32::Args a{};
  a.q = static_cast<const float*>(q);
  a.k = static_cast<const float*>(k);
  a.v = static_cast<const float*>(v);
  a.out = static_cast<const float*>(out);
  a.lse = lse_pad;
  a.dout = static_cast<const float*>(dout);
  a.D = Drow;
  a.dq = static_cast<float*>(dq);
  a.dk = static_cast<float*>(dk);
  a.dv = static_cast<float*>(dv);
  a.B = c.n_seq;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.S = c.S;
  a.S_pad = S_pad;
  a.scale = c.scale;
  a.sched = s;
  if (c.d == 64) {
    if ((r = ensure_smem(f32::attn_bwd_f32<64>, f32::bwd_smem<64>(), 4)) != LCA_OK) return r;
    f32::attn_bwd_f32<64><<<grid, f32::kThreads, f32::bwd_smem<64>(), st>>>(a);
  } else {
    if ((r = ensure_smem(f32::attn_bwd_f32<128>, f32::bwd_smem<128>(), 5)) != LCA_OK) return r;
    f32::attn_bwd_f32<128><<<grid, f32::kThreads, f32::bwd_smem<128>(), st>>>(a);
  }
  return launched("attn_bwd_f32");
}

// ---------------------------------------------------------------- S2-Attn, any group
// Groups whose half is not a whole number of tiles cannot be remapped in
// tile coordinates (a shifted tile would wrap around the end of the
// sequence inside one TMA box).  Then the heads are rolled into the
// workspace in position order (shifted heads by group/2, the others
// copied), the groups become a packed batch of B*S/group sequences of
// `group` tokens for the packed kernels, and results are rolled back.
struct S2Plan {
  bool aligned;          // group/2 is a whole number of tiles: tile remap
  int half;              // group / 2
  int first_q, first_kv; // first shifted query / key-value head
  int n_seq;             // B * S / group
  int64_t group;
};

lca_status plan_s2(const Common& c, int64_t group, int64_t shift_heads, S2Plan* p) {
  if (group <= 0 || group % 2 || c.S % group)
    return fail(LCA_ERR_INVALID_ARG, "group must be even and divide S");
  if (shift_heads < 0 || shift_heads > c.Hq)
    return fail(LCA_ERR_INVALID_ARG, "shift_heads outside [0, Hq]");
  const int rep = c.Hq / c.Hkv;
  if ((c.Hq - shift_heads) % rep)
    return fail(LCA_ERR_INVALID_ARG, "shifted heads must cover whole grouped-query groups");
  p->aligned = (group / 2) % c.tile == 0;
  p->half = static_cast<int>(group / 2);
  p->first_q = static_cast<int>(c.Hq - shift_heads);
  p->first_kv = p->first_q / rep;
  p->n_seq = static_cast<int>(static_cast<int64_t>(c.B) * c.S / group);
  p->group = group;
  return LCA_OK;
}

// The packed problem the rolled tensors form: one token axis of B*S rows,
// n_seq sequences of `group` tokens.
Common packed_of(const Common& c, const S2Plan& p, const int* cu) {
  Common q = c;
  q.n_seq = p.n_seq;
  q.S = c.B * c.S;
  q.S_kv = q.S;  // the rolled keys share the packed token axis
  q.B = 1;
  q.S_seq = static_cast<int>(p.group);
  q.cu = cu;
  return q;
}

size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// Workspace regions of the rolled path, in order.
struct S2Work {
  size_t cu, q, kv, lse;  // bytes of the offsets, a query-side and a kv-side tensor, lse
};
S2Work s2_work(const Common& c, const S2Plan& p) {
  const size_t e = c.dtype == LCA_BF16 ? 2 : 4;
  const size_t rows = static_cast<size_t>(c.B) * c.S;
  return {align256(static_cast<size_t>(p.n_seq + 1) * 4), align256(rows * c.Hq * c.d * e),
          align256(rows * c.Hkv * c.d * e), align256(rows * c.Hq * 4)};
}
size_t s2_fwd_ws_bytes(const Common& c, const S2Plan& p) {
  if (p.aligned) return 0;
  const S2Work w = s2_work(c, p);
  return w.cu + 2 * w.q + 2 * w.kv + w.lse;  // cu | q | k | v | out | lse
}
size_t s2_bwd_ws_bytes(const Common& c, const S2Plan& p) {
  if (p.aligned) return ws_bytes_of(c);
  const S2Work w = s2_work(c, p);
  // cu | q | k | v | out | dout | lse | dq | dk | dv | the packed backward's own
  return w.cu + 4 * w.q + 4 * w.kv + w.lse + ws_bytes_of(packed_of(c, p, nullptr));
}

template <bool kScatter>
lca_status roll_rows(const void* src, void* dst, const Common& c, int H, int first, int half,
                     cudaStream_t st) {
  const int e = c.dtype == LCA_BF16 ? 2 : 4;
  const int vec = c.d * e / 16;
  const int64_t n = static_cast<int64_t>(c.B) * c.S * H * vec;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 148 * 16));
  s2_roll_rows<kScatter><<<blocks, 256, 0, st>>>(static_cast<const uint4*>(src),
                                                 static_cast<uint4*>(dst), c.B, c.S, H, first,
                                                 half, vec);
  return launched("s2_roll_rows");
}

template <bool kScatter>
lca_status roll_lse(const float* src, float* dst, const Common& c, int first, int half,
                    cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(c.B) * c.S * c.Hq;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 148 * 16));
  s2_roll_lse<kScatter><<<blocks, 256, 0, st>>>(src, dst, c.B, c.S, c.Hq, first, half);
  return launched("s2_roll_lse");
}

lca_status s2_fwd_rolled(const Common& c, const S2Plan& p, int causal, const void* q,
                         const void* k, const void* v, void* out, float* lse, void* ws,
                         size_t ws_bytes, cudaStream_t st) {
  if (!ws) return fail(LCA_ERR_WORKSPACE, "workspace is NULL (group/2 is not a whole number of tiles)");
  if (ws_bytes < s2_fwd_ws_bytes(c, p))
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes,
                s2_fwd_ws_bytes(c, p));
  if (!aligned16(ws)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  const S2Work w = s2_work(c, p);
  char* b = static_cast<char*>(ws);
  int* cu = reinterpret_cast<int*>(b);
  void* qr = b + w.cu;
  void* kr = b + w.cu + w.q;
  void* vr = b + w.cu + w.q + w.kv;
  void* outr = b + w.cu + w.q + 2 * w.kv;
  float* lser = reinterpret_cast<float*>(b + w.cu + 2 * w.q + 2 * w.kv);
  fill_offsets<<<(p.n_seq + 256) / 256, 256, 0, st>>>(cu, p.n_seq, static_cast<int>(p.group));
  lca_status r;
  if ((r = launched("fill_offsets")) != LCA_OK) return r;
  if ((r = roll_rows<false>(q, qr, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(k, kr, c, c.Hkv, p.first_kv, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(v, vr, c, c.Hkv, p.first_kv, p.half, st)) != LCA_OK) return r;
  const Common pc = packed_of(c, p, cu);
  AttnSched s;
  if ((r = make_chunk_sched(pc, causal, 0, nullptr, &s)) != LCA_OK) return r;
  if ((r = run_fwd(pc, s, qr, kr, vr, outr, lser, kDefaultBudget, st)) != LCA_OK) return r;
  if ((r = roll_rows<true>(outr, out, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  return roll_lse<true>(lser, lse, c, p.first_q, p.half, st);
}

lca_status s2_bwd_rolled(const Common& c, const S2Plan& p, int causal, const void* q,
                         const void* k, const void* v, const void* out, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* ws,
                         size_t ws_bytes, cudaStream_t st) {
  if (!ws) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  if (ws_bytes < s2_bwd_ws_bytes(c, p))
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes,
                s2_bwd_ws_bytes(c, p));
  if (!aligned16(ws)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  const S2Work w = s2_work(c, p);
  char* b = static_cast<char*>(ws);
  size_t o = 0;
  int* cu = reinterpret_cast<int*>(b + o);
  o += w.cu;
  void* qr = b + o;
  o += w.q;
  void* kr = b + o;
  o += w.kv;
  void* vr = b + o;
  o += w.kv;
  void* outr = b + o;
  o += w.q;
  void* dor = b + o;
  o += w.q;
  float* lser = reinterpret_cast<float*>(b + o);
  o += w.lse;
  void* dqr = b + o;
  o += w.q;
  void* dkr = b + o;
  o += w.kv;
  void* dvr = b + o;
  o += w.kv;
  void* rest = b + o;
  fill_offsets<<<(p.n_seq + 256) / 256, 256, 0, st>>>(cu, p.n_seq, static_cast<int>(p.group));
  lca_status r;
  if ((r = launched("fill_offsets")) != LCA_OK) return r;
  if ((r = roll_rows<false>(q, qr, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(k, kr, c, c.Hkv, p.first_kv, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(v, vr, c, c.Hkv, p.first_kv, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(out, outr, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<false>(dout, dor, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  if ((r = roll_lse<false>(lse, lser, c, p.first_q, p.half, st)) != LCA_OK) return r;
  const Common pc = packed_of(c, p, cu);
  AttnSched s;
  if ((r = make_chunk_sched(pc, causal, 0, nullptr, &s)) != LCA_OK) return r;
  if ((r = run_bwd(pc, s, qr, kr, vr, outr, lser, dor, dqr, dkr, dvr, rest, ws_bytes - o,
                   kDefaultBudget, st)) != LCA_OK)
    return r;
  if ((r = roll_rows<true>(dqr, dq, c, c.Hq, p.first_q, p.half, st)) != LCA_OK) return r;
  if ((r = roll_rows<true>(dkr, dk, c, c.Hkv, p.first_kv, p.half, st)) != LCA_OK) return r;
  return roll_rows<true>(dvr, dv, c, c.Hkv, p.first_kv, p.half, st);
}

// ---------------------------------------------------------------- feedforward
lca_status check_ffn(const lca_ffn_shape* sh, int64_t* block) {
  if (!sh) return fail(LCA_ERR_INVALID_ARG, "shape is NULL");
  if (sh->T <= 0 || sh->h <= 0 || sh->f <= 0)
    return fail(LCA_ERR_INVALID_ARG, "dimensions must be positive");
  if (sh->T > (1ll << 31) - 1 || sh->h > (1 << 20) || sh->f > (1 << 20))
    return fail(LCA_ERR_INVALID_ARG, "dimension too large");
  if (sh->h % ffn::kBN || sh->f % 128)
    return fail(LCA_ERR_UNSUPPORTED, "feedforward needs h %% 256 == 0 and f %% 128 == 0");
  int64_t b = *block;
  if (b < 0 || b % ffn::kBM)
    return fail(LCA_ERR_INVALID_ARG, "block_tokens must be a non-negative multiple of 128");
  const int64_t t_pad = (sh->T + ffn::kBM - 1) / ffn::kBM * ffn::kBM;
  if (b == 0) b = LCA_FFN_BLOCK_DEFAULT;
  if (b > t_pad) b = t_pad;
  *block = b;
  return LCA_OK;
}

// Band heights of the feedforward tile raster (row tiles).  Products whose B
// (weight) operand is the large one and is swept column by column take
// bands of 32 row tiles, so every weight column is read from DRAM twice per
// 8192-row block while the band's A rows (32 MB) stay in L2; products whose B
// fits in L2 whole (W_down for the down product, the block's x for the
// weight gradients) go row tile by row tile, so B stays resident and A is
// read once.  Measured on the Llama-2-7B feedforward (32K tokens): bands of
// 32 / 1 run as fast as 16 / 16 (forward 1450 vs 1448 TFLOP/s, backward 1122
// vs 1129); a band of the whole block for the weight products was slower
// (1349 / 1095: the block's 64 MB of rows do not stay in L2).
constexpr int kFfnBandWide = 32;
constexpr int kFfnBandNarrow = 1;

template <int kEpi, bool kAmn, bool kBmn, bool kSplit>
lca_status launch_ffn_gemm(const CUtensorMap& ma0, const CUtensorMap& ma1, const CUtensorMap& mb0,
                           const CUtensorMap& mb1, const ffn::Args& a0, int slot,
                           cudaStream_t st) {
  auto kernel = ffn_gemm_sm100<kEpi, kAmn, kBmn, kSplit>;
  if (a0.group_m < 1) return fail(LCA_ERR_INVALID_ARG, "internal: feedforward band height < 1");
  ffn::Args a = a0;
  if (a.group_m > a.n_tm) a.group_m = a.n_tm;  // one band at most (keeps t / (gm * n_tn) small)
  lca_status r = ensure_smem(kernel, ffn::kSmemBytes, slot);
  if (r != LCA_OK) return r;
  int sms = 0;
  if ((r = sm_count(&sms)) != LCA_OK) return r;
  const int tiles = a.n_tm * a.n_tn;
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  kernel<<<grid, ffn::kThreads, ffn::kSmemBytes, st>>>(ma0, ma1, mb0, mb1, a);
  return launched("ffn_gemm_sm100");
}

// ---------------------------------------------------------------- feedforward blocks
// The products of one block of token rows [r0, r0 + rows) of the
// feedforward, over tensor maps made once per call (x, dout and the
// outputs span all T rows; the intermediates span one block).
struct FfnFwdPlan {
  CUtensorMap mx, mg, mu, md, mh;
  int64_t h, f;
  void* out;
  void* H;
};

lca_status ffn_fwd_plan(const void* x, const void* w_gate, const void* w_up, const void* w_down,
                        int64_t T, int64_t h, int64_t f, int64_t block, void* out, void* H,
                        FfnFwdPlan* p) {
  lca_status r;
  if ((r = make_map_2d(&p->mx, x, T, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->mg, w_gate, f, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->mu, w_up, f, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->md, w_down, h, f)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->mh, H, block, f)) != LCA_OK) return r;
  p->h = h;
  p->f = f;
  p->out = out;
  p->H = H;
  return LCA_OK;
}

lca_status ffn_fwd_rows(const FfnFwdPlan& p, int64_t r0, int rows, cudaStream_t st) {
  const int64_t h = p.h, f = p.f;
  lca_status r;
  ffn::Args g1{};
  g1.M = rows;
  g1.K = static_cast<int>(h);
  g1.n_tm = (rows + ffn::kBM - 1) / ffn::kBM;
  g1.n_tn = static_cast<int>(f / 128);
  g1.a_off = static_cast<int>(r0);
  g1.ldo = static_cast<int>(f);
  g1.budget = kDefaultBudget;
  g1.group_m = kFfnBandWide;
  g1.out = static_cast<__nv_bfloat16*>(p.H);
  if ((r = launch_ffn_gemm<ffn::EPI_SWIGLU, false, false, false>(p.mx, p.mx, p.mg, p.mu, g1, 7,
                                                                 st)) != LCA_OK)
    return r;
  ffn::Args g2{};
  g2.M = rows;
  g2.K = static_cast<int>(f);
  g2.n_tm = g1.n_tm;
  g2.n_tn = static_cast<int>(h / ffn::kBN);
  g2.a_off = 0;
  g2.ldo = static_cast<int>(h);
  g2.budget = kDefaultBudget;
  g2.group_m = kFfnBandNarrow;
  g2.out = static_cast<__nv_bfloat16*>(p.out) + r0 * h;
  return launch_ffn_gemm<ffn::EPI_STORE, false, false, false>(p.mh, p.mh, p.md, p.md, g2, 8, st);
}

struct FfnBwdPlan {
  // K-major views (boxes of 128 rows) and MN-major views (boxes of 64 rows)
  CUtensorMap x_k, x_mn, do_k, do_mn, wg_k, wu_k, wg_mn, wu_mn, wd_mn, dg_k, du_k, dgu_mn, h_mn;
  int64_t h, f;
  __nv_bfloat16 *dH, *dGU, *H;
  float *dw_gate, *dw_up, *dw_down;
};

// ws: dH [block, f] | [dG | dU] [block, 2f] | H [block, f], bf16
lca_status ffn_bwd_plan(const void* x, const void* w_gate, const void* w_up, const void* w_down,
                        const void* dout, int64_t T, int64_t h, int64_t f, int64_t block,
                        float* dw_gate, float* dw_up, float* dw_down, void* workspace,
                        FfnBwdPlan* p) {
  auto* ws = static_cast<__nv_bfloat16*>(workspace);
  p->dH = ws;
  p->dGU = ws + block * f;
  p->H = ws + 3 * block * f;
  p->h = h;
  p->f = f;
  p->dw_gate = dw_gate;
  p->dw_up = dw_up;
  p->dw_down = dw_down;
  lca_status r;
  if ((r = make_map_2d(&p->x_k, x, T, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->x_mn, x, T, h, 64)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->do_k, dout, T, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->do_mn, dout, T, h, 64)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->wg_k, w_gate, f, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->wu_k, w_up, f, h)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->wg_mn, w_gate, f, h, 64)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->wu_mn, w_up, f, h, 64)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->wd_mn, w_down, h, f, 64)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->dg_k, p->dGU, block, f, 128, 2 * f)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->du_k, p->dGU + f, block, f, 128, 2 * f)) != LCA_OK) return r;
  if ((r = make_map_2d(&p->dgu_mn, p->dGU, block, 2 * f, 64)) != LCA_OK) return r;
  return make_map_2d(&p->h_mn, p->H, block, f, 64);
}

// dx_rows: where row r0 of dx goes (the plan's dx + r0 * h for a whole-T
// dx; a block-sized buffer for a caller that consumes dx block by block).
lca_status ffn_bwd_rows(const FfnBwdPlan& p, int64_t r0, int rows, void* dx_rows,
                        cudaStream_t st) {
  const int64_t h = p.h, f = p.f;
  const int n_tm = (rows + ffn::kBM - 1) / ffn::kBM;
  const int k_rows = (rows + ffn::kBK - 1) / ffn::kBK * ffn::kBK;  // whole K steps
  lca_status r;
  ffn::Args g{};
  g.budget = kDefaultBudget;
  // dH = dout W_down
  g.M = rows, g.K = static_cast<int>(h), g.n_tm = n_tm, g.n_tn = static_cast<int>(f / ffn::kBN);
  g.group_m = kFfnBandWide;
  g.a_off = static_cast<int>(r0), g.b_off = 0, g.ldo = static_cast<int>(f), g.out = p.dH;
  if ((r = launch_ffn_gemm<ffn::EPI_STORE, false, true, false>(p.do_k, p.do_k, p.wd_mn, p.wd_mn,
                                                               g, 9, st)) != LCA_OK)
    return r;
  // G, U recomputed; dG, dU, H written
  g = ffn::Args{};
  g.budget = kDefaultBudget;
  g.M = rows, g.K = static_cast<int>(h), g.n_tm = n_tm, g.n_tn = static_cast<int>(f / 128);
  g.group_m = kFfnBandWide;
  g.a_off = static_cast<int>(r0), g.b_off = 0, g.ldo = static_cast<int>(2 * f);
  g.ldo3 = static_cast<int>(f), g.ld_in = static_cast<int>(f), g.in = p.dH;
  g.out = p.dGU, g.out2 = p.dGU + f, g.out3 = p.H;
  if ((r = launch_ffn_gemm<ffn::EPI_SWIGLU_BWD, false, false, false>(p.x_k, p.x_k, p.wg_k, p.wu_k,
                                                                     g, 10, st)) != LCA_OK)
    return r;
  // dX = dG W_gate + dU W_up
  g = ffn::Args{};
  g.budget = kDefaultBudget;
  g.M = rows, g.K = static_cast<int>(2 * f), g.n_tm = n_tm, g.n_tn = static_cast<int>(h / ffn::kBN);
  g.group_m = kFfnBandNarrow;
  g.a_off = 0, g.b_off = 0, g.ldo = static_cast<int>(h);
  g.out = static_cast<__nv_bfloat16*>(dx_rows);
  if ((r = launch_ffn_gemm<ffn::EPI_STORE, false, true, true>(p.dg_k, p.du_k, p.wg_mn, p.wu_mn, g,
                                                              11, st)) != LCA_OK)
    return r;
  // [dW_gate; dW_up] += [dG | dU]^T x: one product, rows split at f
  g = ffn::Args{};
  g.budget = kDefaultBudget;
  g.M = static_cast<int>(2 * f), g.K = k_rows, g.n_tm = static_cast<int>(2 * f / ffn::kBM);
  g.group_m = kFfnBandNarrow;
  g.n_tn = static_cast<int>(h / ffn::kBN);
  g.a_off = 0, g.b_off = static_cast<int>(r0), g.ldo = static_cast<int>(h);
  g.m_split = static_cast<int>(f), g.out32 = p.dw_gate, g.out32b = p.dw_up;
  if ((r = launch_ffn_gemm<ffn::EPI_ACC32, true, true, false>(p.dgu_mn, p.dgu_mn, p.x_mn, p.x_mn,
                                                              g, 12, st)) != LCA_OK)
    return r;
  // dW_down += dout^T H
  g.M = static_cast<int>(h), g.m_split = static_cast<int>(h), g.out32b = nullptr;
  g.group_m = kFfnBandWide;
  g.n_tm = static_cast<int>(h / ffn::kBM);
  g.n_tn = static_cast<int>(f / ffn::kBN);
  g.a_off = static_cast<int>(r0), g.b_off = 0, g.ldo = static_cast<int>(f), g.out32 = p.dw_down;
  return launch_ffn_gemm<ffn::EPI_ACC32, true, true, false>(p.do_mn, p.do_mn, p.h_mn, p.h_mn, g,
                                                            12, st);
}

// ---------------------------------------------------------------- blocks
// A query block of Sq rows at position q_pos0 against a key/value block of
// Sk keys at position k_pos0 (a sequence-parallel ring step).
lca_status check_block(const lca_block_shape* sh, Common* c) {
  if (!sh) return fail(LCA_ERR_INVALID_ARG, "shape is NULL");
  const lca_shape one{sh->B, sh->Hq, sh->Hkv, sh->Sq, sh->d, sh->dtype, sh->scale};
  lca_status r = check_shape(&one, c);
  if (r != LCA_OK) return r;
  if (sh->Sk <= 0) return fail(LCA_ERR_INVALID_ARG, "dimensions must be positive");
  if (sh->Sk > (1ll << 26)) return fail(LCA_ERR_INVALID_ARG, "dimension too large");
  if (sh->B * sh->Sk > (1ll << 31) - 1)
    return fail(LCA_ERR_INVALID_ARG, "B*Sk must fit in 31 bits");
  if (c->dtype != LCA_BF16)
    return fail(LCA_ERR_UNSUPPORTED, "block calls run on the bf16 tensor-core path only");
  c->S_kv = static_cast<int>(sh->Sk);
  return LCA_OK;
}

enum { REL_NONE = 0, REL_FULL = 1, REL_CAUSAL = 2 };

// Which keys of the block the queries see: all (REL_FULL), none (REL_NONE)
// or a causal band whose diagonal key tile for query tile Q is Q + *diag.
lca_status block_relation(const Common& c, int causal, int64_t q_pos0, int64_t k_pos0, int* rel,
                          int* diag) {
  if (q_pos0 < 0 || k_pos0 < 0 || q_pos0 > (1ll << 40) || k_pos0 > (1ll << 40))
    return fail(LCA_ERR_INVALID_ARG, "block positions must lie in [0, 2^40]");
  *diag = 0;
  if (!causal || k_pos0 + c.S_kv - 1 <= q_pos0) {
    *rel = REL_FULL;
  } else if (k_pos0 > q_pos0 + c.S - 1) {
    *rel = REL_NONE;
  } else {
    if ((q_pos0 - k_pos0) % c.tile)
      return fail(LCA_ERR_INVALID_ARG,
                  "causal blocks that overlap on the diagonal must start a multiple of %d "
                  "positions apart",
                  c.tile);
    *rel = REL_CAUSAL;
    *diag = static_cast<int>((q_pos0 - k_pos0) / c.tile);
  }
  return LCA_OK;
}

// The schedule of one block: one chunk spanning the key block, in order.
// REL_NONE becomes a causal band with its diagonal before every key tile
// (no query sees a key), which the kernels turn into empty results.
void make_block_sched(const Common& c, int rel, int diag, AttnSched* s) {
  std::memset(s, 0, sizeof *s);
  s->S = c.S;
  s->tile = c.tile;
  s->n_tiles = (c.S + c.tile - 1) / c.tile;
  s->S_kv = c.S_kv;
  s->n_kv_tiles = (c.S_kv + c.tile - 1) / c.tile;
  s->causal = rel != REL_FULL;
  s->diag = rel == REL_NONE ? -(s->n_tiles + 1) : diag;
  s->kv_chunk = c.S_kv;
  s->n_chunks = 1;
  s->order = LCA_ORDER_INORDER;
  s->q_block = c.S;
}

// ---------------------------------------------------------------- blockwise transformer
// One sweep of the Blockwise Transformer over the query blocks: per block,
// the attention of its rows over the keys they see, then the feedforward of
// those rows.
struct BptPlan {
  Common attn;     // shape of a full query block (rows == q_block)
  int64_t S, h, f, qb;
  int causal;
};

lca_status check_bpt(const lca_bpt_shape* sh, int backward, BptPlan* p) {
  if (!sh) return fail(LCA_ERR_INVALID_ARG, "shape is NULL");
  if (sh->S <= 0 || sh->Hq <= 0 || sh->Hkv <= 0 || sh->d <= 0 || sh->f <= 0)
    return fail(LCA_ERR_INVALID_ARG, "dimensions must be positive");
  const int64_t qb = sh->q_block ? sh->q_block : LCA_FFN_BLOCK_DEFAULT;
  if (qb <= 0 || qb % 128) return fail(LCA_ERR_INVALID_ARG, "q_block must be a positive multiple of 128");
  const lca_block_shape bs{1, sh->Hq, sh->Hkv, qb < sh->S ? qb : sh->S, sh->S, sh->d, LCA_BF16,
                           sh->scale};
  lca_status r = check_block(&bs, &p->attn);
  if (r != LCA_OK) return r;
  const lca_ffn_shape fs{sh->S, sh->Hq * sh->d, sh->f};
  int64_t blk = qb;
  if ((r = check_ffn(&fs, &blk)) != LCA_OK) return r;
  if (backward && sh->f % ffn::kBN)
    return fail(LCA_ERR_UNSUPPORTED, "feedforward backward needs f %% 256 == 0");
  p->S = sh->S;
  p->h = sh->Hq * sh->d;
  p->f = sh->f;
  p->qb = qb;
  return LCA_OK;
}

// Attention shape and schedule of the query block [r0, r0 + rows): its
// rows against keys [0, r0 + rows) (causal) or all keys.
void bpt_block(const BptPlan& p, int causal, int64_t r0, int rows, Common* c, AttnSched* s) {
  *c = p.attn;
  c->S = rows;
  c->S_seq = rows;
  c->S_kv = static_cast<int>(causal ? r0 + rows : p.S);
  int rel, diag;
  block_relation(*c, causal, r0, 0, &rel, &diag);  // r0 is a multiple of the tile
  make_block_sched(*c, rel, diag, s);
}

size_t bpt_fwd_ws(const BptPlan& p) {
  return align256(static_cast<size_t>(p.attn.Hq) * p.qb * 4) +
         static_cast<size_t>(p.qb) * p.f * 2;  // lse of a block | H of a block
}

size_t bpt_bwd_ws(const BptPlan& p) {
  Common c = p.attn;  // a full block
  const size_t kv = static_cast<size_t>(p.S) * p.attn.Hkv * p.attn.d * 4;
  return 4 * static_cast<size_t>(p.qb) * p.f * 2           // feedforward backward
         + align256(static_cast<size_t>(p.qb) * p.h * 2)    // d(attention out) of a block
         + align256(ws_bytes_of(c))                          // attention backward of a block
         + align256(static_cast<size_t>(p.attn.Hq) * p.qb * 4)  // lse of a block
         + 2 * align256(kv);                                 // dk, dv accumulators
}

}  // namespace

extern "C" {

const char* lca_status_string(lca_status s) {
  switch (s) {
    case LCA_OK: return "LCA_OK";
    case LCA_ERR_INVALID_ARG: return "LCA_ERR_INVALID_ARG";
    case LCA_ERR_UNSUPPORTED: return "LCA_ERR_UNSUPPORTED";
    case LCA_ERR_CUDA: return "LCA_ERR_CUDA";
    case LCA_ERR_TIMEOUT: return "LCA_ERR_TIMEOUT";
    case LCA_ERR_WORKSPACE: return "LCA_ERR_WORKSPACE";
  }
  return "LCA_ERR_UNKNOWN";
}

const char* lca_last_error(void) { return t_last_error.c_str(); }

int lca_version(void) { return (1 << 16) | 0; }

lca_status lca_attn_fwd(const lca_shape* shape, const void* q, const void* k, const void* v,
                        int causal, int64_t kv_chunk, const lca_opts* opts, void* out,
                        float* lse, void* stream) {
  Common c;
  lca_status r = check_shape(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse})) != LCA_OK) return r;
  AttnSched s;
  if ((r = make_chunk_sched(c, causal, kv_chunk, opts, &s)) != LCA_OK) return r;
  return run_fwd(c, s, q, k, v, out, lse, budget_of(opts), static_cast<cudaStream_t>(stream));
}

size_t lca_attn_bwd_workspace_size(const lca_shape* shape) {
  Common c;
  const std::string keep = t_last_error;  // a size query leaves the error detail alone
  const bool ok = check_shape(shape, &c) == LCA_OK;
  t_last_error = keep;
  return ok ? ws_bytes_of(c) : 0;
}

lca_status lca_attn_bwd(const lca_shape* shape, const void* q, const void* k, const void* v,
                        const void* out, const float* lse, const void* dout, int causal,
                        void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                        void* stream) {
  Common c;
  lca_status r = check_shape(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse, dout, dq, dk, dv})) != LCA_OK) return r;
  AttnSched s;
  if ((r = make_chunk_sched(c, causal, 0, nullptr, &s)) != LCA_OK) return r;
  return run_bwd(c, s, q, k, v, out, lse, dout, dq, dk, dv, workspace, ws_bytes, kDefaultBudget,
                 static_cast<cudaStream_t>(stream));
}

lca_status lca_s2attn_fwd(const lca_shape* shape, const void* q, const void* k, const void* v,
                          int causal, int64_t group, int64_t shift_heads, void* out, float* lse,
                          void* stream) {
  return lca_s2attn_fwd_ws(shape, q, k, v, causal, group, shift_heads, out, lse, nullptr, 0,
                           stream);
}

size_t lca_s2attn_fwd_workspace_size(const lca_shape* shape, int64_t group,
                                     int64_t shift_heads) {
  Common c;
  S2Plan p;
  const std::string keep = t_last_error;
  const bool ok = check_shape(shape, &c) == LCA_OK && plan_s2(c, group, shift_heads, &p) == LCA_OK;
  t_last_error = keep;
  return ok ? s2_fwd_ws_bytes(c, p) : 0;
}

size_t lca_s2attn_bwd_workspace_size(const lca_shape* shape, int64_t group,
                                     int64_t shift_heads) {
  Common c;
  S2Plan p;
  const std::string keep = t_last_error;
  const bool ok = check_shape(shape, &c) == LCA_OK && plan_s2(c, group, shift_heads, &p) == LCA_OK;
  t_last_error = keep;
  return ok ? s2_bwd_ws_bytes(c, p) : 0;
}

lca_status lca_s2attn_fwd_ws(const lca_shape* shape, const void* q, const void* k,
                             const void* v, int causal, int64_t group, int64_t shift_heads,
                             void* out, float* lse, void* workspace, size_t ws_bytes,
                             void* stream) {
  Common c;
  lca_status r = check_shape(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse})) != LCA_OK) return r;
  S2Plan p;
  if ((r = plan_s2(c, group, shift_heads, &p)) != LCA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!p.aligned)
    return s2_fwd_rolled(c, p, causal, q, k, v, out, lse, workspace, ws_bytes, st);
  AttnSched s;
  if ((r = make_s2_sched(c, causal, group, shift_heads, &s)) != LCA_OK) return r;
  return run_fwd(c, s, q, k, v, out, lse, kDefaultBudget, st);
}

lca_status lca_s2attn_bwd(const lca_shape* shape, const void* q, const void* k, const void* v,
                          const void* out, const float* lse, const void* dout, int causal,
                          int64_t group, int64_t shift_heads, void* dq, void* dk, void* dv,
                          void* workspace, size_t ws_bytes, void* stream) {
  Common c;
  lca_status r = check_shape(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse, dout, dq, dk, dv})) != LCA_OK) return r;
  S2Plan p;
  if ((r = plan_s2(c, group, shift_heads, &p)) != LCA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!p.aligned)
    return s2_bwd_rolled(c, p, causal, q, k, v, out, lse, dout, dq, dk, dv, workspace, ws_bytes,
                         st);
  AttnSched s;
  if ((r = make_s2_sched(c, causal, group, shift_heads, &s)) != LCA_OK) return r;
  return run_bwd(c, s, q, k, v, out, lse, dout, dq, dk, dv, workspace, ws_bytes, kDefaultBudget,
                 st);
}

lca_status lca_attn_fwd_varlen(const lca_shape* shape, const int32_t* cu_seqlens,
                               int64_t max_seqlen, const void* q, const void* k, const void* v,
                               int causal, int64_t kv_chunk, const lca_opts* opts, void* out,
                               float* lse, void* stream) {
  Common c;
  lca_status r = check_packed(shape, cu_seqlens, max_seqlen, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse})) != LCA_OK) return r;
  AttnSched s;
  if ((r = make_chunk_sched(c, causal, kv_chunk, opts, &s)) != LCA_OK) return r;
  return run_fwd(c, s, q, k, v, out, lse, budget_of(opts), static_cast<cudaStream_t>(stream));
}

size_t lca_attn_bwd_varlen_workspace_size(const lca_shape* shape, int64_t max_seqlen) {
  Common c;
  const std::string keep = t_last_error;
  // the offsets are not read here; any aligned non-null stand-in passes the check
  static const int32_t stand_in[1] = {0};
  const bool ok = check_packed(shape, stand_in, max_seqlen, &c) == LCA_OK;
  t_last_error = keep;
  return ok ? ws_bytes_of(c) : 0;
}

lca_status lca_attn_bwd_varlen(const lca_shape* shape, const int32_t* cu_seqlens,
                               int64_t max_seqlen, const void* q, const void* k, const void* v,
                               const void* out, const float* lse, const void* dout, int causal,
                               void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                               void* stream) {
  Common c;
  lca_status r = check_packed(shape, cu_seqlens, max_seqlen, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse, dout, dq, dk, dv})) != LCA_OK) return r;
  AttnSched s;
  if ((r = make_chunk_sched(c, causal, 0, nullptr, &s)) != LCA_OK) return r;
  return run_bwd(c, s, q, k, v, out, lse, dout, dq, dk, dv, workspace, ws_bytes, kDefaultBudget,
                 static_cast<cudaStream_t>(stream));
}

size_t lca_ffn_workspace_size(const lca_ffn_shape* shape, int64_t block_tokens) {
  const std::string keep = t_last_error;  // a size query leaves the error detail alone
  int64_t b = block_tokens;
  const bool ok = check_ffn(shape, &b) == LCA_OK;
  t_last_error = keep;
  return ok ? static_cast<size_t>(b) * static_cast<size_t>(shape->f) * 2 : 0;
}

lca_status lca_ffn_fwd(const lca_ffn_shape* shape, const void* x, const void* w_gate,
                       const void* w_up, const void* w_down, int64_t block_tokens, void* out,
                       void* workspace, size_t ws_bytes, void* stream) {
  int64_t block = block_tokens;
  lca_status r = check_ffn(shape, &block);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({x, w_gate, w_up, w_down, out})) != LCA_OK) return r;
  if (!workspace) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  const size_t need = static_cast<size_t>(block) * static_cast<size_t>(shape->f) * 2;
  if (ws_bytes < need)
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
  if (!aligned16(workspace)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  FfnFwdPlan p;
  if ((r = ffn_fwd_plan(x, w_gate, w_up, w_down, shape->T, shape->h, shape->f, block, out,
                        workspace, &p)) != LCA_OK)
    return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int64_t r0 = 0; r0 < shape->T; r0 += block) {
    const int rows = static_cast<int>(shape->T - r0 < block ? shape->T - r0 : block);
    if ((r = ffn_fwd_rows(p, r0, rows, st)) != LCA_OK) return r;
  }
  return LCA_OK;
}

size_t lca_ffn_bwd_workspace_size(const lca_ffn_shape* shape, int64_t block_tokens) {
  const std::string keep = t_last_error;
  int64_t b = block_tokens;
  const bool ok = check_ffn(shape, &b) == LCA_OK && shape->f % ffn::kBN == 0;
  t_last_error = keep;
  // dH, dG, dU and H, each [block, f] bf16
  return ok ? 4 * static_cast<size_t>(b) * static_cast<size_t>(shape->f) * 2 : 0;
}

lca_status lca_ffn_bwd(const lca_ffn_shape* shape, const void* x, const void* w_gate,
                       const void* w_up, const void* w_down, const void* dout,
                       int64_t block_tokens, void* dx, float* dw_gate, float* dw_up,
                       float* dw_down, void* workspace, size_t ws_bytes, void* stream) {
  int64_t block = block_tokens;
  lca_status r = check_ffn(shape, &block);
  if (r != LCA_OK) return r;
  if (shape->f % ffn::kBN)
    return fail(LCA_ERR_UNSUPPORTED, "feedforward backward needs f %% 256 == 0");
  if ((r = check_ptrs({x, w_gate, w_up, w_down, dout, dx, dw_gate, dw_up, dw_down})) != LCA_OK)
    return r;
  if (!workspace) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  const size_t one = static_cast<size_t>(block) * static_cast<size_t>(shape->f) * 2;
  if (ws_bytes < 4 * one)
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, 4 * one);
  if (!aligned16(workspace)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  FfnBwdPlan p;
  if ((r = ffn_bwd_plan(x, w_gate, w_up, w_down, dout, shape->T, shape->h, shape->f, block,
                        dw_gate, dw_up, dw_down, workspace, &p)) != LCA_OK)
    return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int64_t r0 = 0; r0 < shape->T; r0 += block) {
    const int rows = static_cast<int>(shape->T - r0 < block ? shape->T - r0 : block);
    if ((r = ffn_bwd_rows(p, r0, rows, static_cast<__nv_bfloat16*>(dx) + r0 * shape->h, st)) !=
        LCA_OK)
      return r;
  }
  return LCA_OK;
}

lca_status lca_lse_merge(int64_t rows, int64_t d, const float* o_a, const float* lse_a,
                         const float* o_b, const float* lse_b, float* o_out, float* lse_out,
                         void* stream) {
  if (rows <= 0 || d <= 0 || d > (1 << 20))
    return fail(LCA_ERR_INVALID_ARG, "rows and d must be positive");
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out)
    return fail(LCA_ERR_INVALID_ARG, "NULL pointer");
  const int64_t warps_needed = rows;
  const unsigned blocks =
      static_cast<unsigned>(std::min<int64_t>((warps_needed * 32 + 255) / 256, 148 * 32));
  lse_merge_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      rows, static_cast<int>(d), o_a, lse_a, o_b, lse_b, o_out, lse_out);
  return launched("lse_merge_kernel");
}

lca_status lca_attn_fwd_block(const lca_block_shape* shape, const void* q, const void* k,
                              const void* v, int causal, int64_t q_pos0, int64_t k_pos0,
                              int accumulate, float* o_acc, float* lse_acc, void* out,
                              void* stream) {
  Common c;
  lca_status r = check_block(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, lse_acc})) != LCA_OK) return r;
  if (!o_acc && !out) return fail(LCA_ERR_INVALID_ARG, "o_acc and out are both NULL");
  if (accumulate && !o_acc)
    return fail(LCA_ERR_INVALID_ARG, "accumulating needs the running o_acc");
  if ((o_acc && !aligned16(o_acc)) || (out && !aligned16(out)))
    return fail(LCA_ERR_INVALID_ARG, "o_acc / out not 16-byte aligned");
  int rel, diag;
  if ((r = block_relation(c, causal, q_pos0, k_pos0, &rel, &diag)) != LCA_OK) return r;
  if (rel == REL_NONE && accumulate && !out) return LCA_OK;  // nothing visible to add
  AttnSched s;
  make_block_sched(c, rel, diag, &s);
  FwdBlock fb;
  fb.block = true;
  fb.o_acc = o_acc;
  fb.accumulate = accumulate ? 1 : 0;
  return run_fwd(c, s, q, k, v, out, lse_acc, kDefaultBudget, static_cast<cudaStream_t>(stream),
                 fb);
}

size_t lca_attn_bwd_block_workspace_size(const lca_block_shape* shape) {
  Common c;
  const std::string keep = t_last_error;
  const bool ok = check_block(shape, &c) == LCA_OK;
  t_last_error = keep;
  return ok ? ws_bytes_of(c) : 0;
}

lca_status lca_attn_bwd_block_prep(const lca_block_shape* shape, const void* out,
                                   const float* lse, const void* dout, void* workspace,
                                   size_t ws_bytes, void* stream) {
  Common c;
  lca_status r = check_block(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({out, lse, dout})) != LCA_OK) return r;
  if ((r = check_ws(c, workspace, ws_bytes)) != LCA_OK) return r;
  return bwd_prep(c, out, lse, dout, workspace, static_cast<cudaStream_t>(stream));
}

lca_status lca_attn_bwd_block(const lca_block_shape* shape, const void* q, const void* k,
                              const void* v, const void* dout, int causal, int64_t q_pos0,
                              int64_t k_pos0, void* workspace, size_t ws_bytes, float* dk_acc,
                              float* dv_acc, int accumulate_kv, void* dk, void* dv,
                              void* stream) {
  Common c;
  lca_status r = check_block(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, dout})) != LCA_OK) return r;
  if ((r = check_ws(c, workspace, ws_bytes)) != LCA_OK) return r;
  const bool acc = dk_acc || dv_acc;
  if (acc == (dk || dv))
    return fail(LCA_ERR_INVALID_ARG, "pass either dk_acc and dv_acc or dk and dv");
  if ((r = acc ? check_ptrs({dk_acc, dv_acc}) : check_ptrs({dk, dv})) != LCA_OK) return r;
  int rel, diag;
  if ((r = block_relation(c, causal, q_pos0, k_pos0, &rel, &diag)) != LCA_OK) return r;
  // no query sees a key: nothing to add (overwriting still writes zeros)
  if (rel == REL_NONE && acc && accumulate_kv) return LCA_OK;
  AttnSched s;
  make_block_sched(c, rel, diag, &s);
  return bwd_main(c, s, q, k, v, dout, workspace, dk, dv, dk_acc, dv_acc, accumulate_kv ? 1 : 0,
                  kDefaultBudget, static_cast<cudaStream_t>(stream));
}

lca_status lca_attn_bwd_block_dq(const lca_block_shape* shape, const void* workspace,
                                 size_t ws_bytes, void* dq, void* stream) {
  Common c;
  lca_status r = check_block(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({dq})) != LCA_OK) return r;
  if ((r = check_ws(c, workspace, ws_bytes)) != LCA_OK) return r;
  return bwd_dq(c, workspace, dq, static_cast<cudaStream_t>(stream));
}

lca_status lca_cast_f32_bf16(int64_t n, const float* src, void* dst, void* stream) {
  if (n <= 0) return fail(LCA_ERR_INVALID_ARG, "n must be positive");
  lca_status r = check_ptrs({src, dst});
  if (r != LCA_OK) return r;
  const int64_t n8 = n / 8;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, 148 * 16));
  cast_f32_bf16<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      src, static_cast<__nv_bfloat16*>(dst), n);
  return launched("cast_f32_bf16");
}

lca_status lca_accumulate_f32(int64_t n, const float* src, float* dst, void* stream) {
  if (n <= 0) return fail(LCA_ERR_INVALID_ARG, "n must be positive");
  lca_status r = check_ptrs({src, dst});
  if (r != LCA_OK) return r;
  const int64_t n4 = n / 4;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256, 148 * 16));
  accumulate_f32<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      src, dst, n);
  return launched("accumulate_f32");
}

size_t lca_bpt_fwd_workspace_size(const lca_bpt_shape* shape) {
  BptPlan p;
  const std::string keep = t_last_error;
  const bool ok = check_bpt(shape, 0, &p) == LCA_OK;
  t_last_error = keep;
  return ok ? bpt_fwd_ws(p) : 0;
}

lca_status lca_bpt_fwd(const lca_bpt_shape* shape, const void* q, const void* k, const void* v,
                       int causal, const void* w_gate, const void* w_up, const void* w_down,
                       void* attn_out, float* lse, void* out, void* workspace, size_t ws_bytes,
                       void* stream) {
  BptPlan p;
  lca_status r = check_bpt(shape, 0, &p);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, w_gate, w_up, w_down, attn_out, lse, out})) != LCA_OK) return r;
  if (!workspace) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  if (ws_bytes < bpt_fwd_ws(p))
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, bpt_fwd_ws(p));
  if (!aligned16(workspace)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* lse_blk = static_cast<float*>(workspace);
  void* H = static_cast<char*>(workspace) + align256(static_cast<size_t>(p.attn.Hq) * p.qb * 4);
  FfnFwdPlan fp;
  if ((r = ffn_fwd_plan(attn_out, w_gate, w_up, w_down, p.S, p.h, p.f, p.qb, out, H, &fp)) !=
      LCA_OK)
    return r;
  const size_t row_q = static_cast<size_t>(p.attn.Hq) * p.attn.d;  // elements per query row
  for (int64_t r0 = 0; r0 < p.S; r0 += p.qb) {
    const int rows = static_cast<int>(p.S - r0 < p.qb ? p.S - r0 : p.qb);
    Common c;
    AttnSched s;
    bpt_block(p, causal, r0, rows, &c, &s);
    FwdBlock fb;
    fb.block = true;
    if ((r = run_fwd(c, s, static_cast<const __nv_bfloat16*>(q) + r0 * row_q, k, v,
                     static_cast<__nv_bfloat16*>(attn_out) + r0 * row_q, lse_blk, kDefaultBudget,
                     st, fb)) != LCA_OK)
      return r;
    const cudaError_t e = cudaMemcpy2DAsync(lse + r0, p.S * sizeof(float), lse_blk,
                                            rows * sizeof(float), rows * sizeof(float),
                                            p.attn.Hq, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy2DAsync(lse of a block)");
    if ((r = ffn_fwd_rows(fp, r0, rows, st)) != LCA_OK) return r;
  }
  return LCA_OK;
}

size_t lca_bpt_bwd_workspace_size(const lca_bpt_shape* shape) {
  BptPlan p;
  const std::string keep = t_last_error;
  const bool ok = check_bpt(shape, 1, &p) == LCA_OK;
  t_last_error = keep;
  return ok ? bpt_bwd_ws(p) : 0;
}

lca_status lca_bpt_bwd(const lca_bpt_shape* shape, const void* q, const void* k, const void* v,
                       int causal, const void* w_gate, const void* w_up, const void* w_down,
                       const void* attn_out, const float* lse, const void* dout, void* dq,
                       void* dk, void* dv, float* dw_gate, float* dw_up, float* dw_down,
                       void* workspace, size_t ws_bytes, void* stream) {
  BptPlan p;
  lca_status r = check_bpt(shape, 1, &p);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, w_gate, w_up, w_down, attn_out, lse, dout, dq, dk, dv, dw_gate,
                       dw_up, dw_down})) != LCA_OK)
    return r;
  if (!workspace) return fail(LCA_ERR_WORKSPACE, "workspace is NULL");
  if (ws_bytes < bpt_bwd_ws(p))
    return fail(LCA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, bpt_bwd_ws(p));
  if (!aligned16(workspace)) return fail(LCA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  void* ffn_ws = w;
  w += 4 * static_cast<size_t>(p.qb) * p.f * 2;
  auto* dx_blk = reinterpret_cast<__nv_bfloat16*>(w);
  w += align256(static_cast<size_t>(p.qb) * p.h * 2);
  void* attn_ws = w;
  w += align256(ws_bytes_of(p.attn));
  float* lse_blk = reinterpret_cast<float*>(w);
  w += align256(static_cast<size_t>(p.attn.Hq) * p.qb * 4);
  const size_t kv_elems = static_cast<size_t>(p.S) * p.attn.Hkv * p.attn.d;
  float* dk_acc = reinterpret_cast<float*>(w);
  w += align256(kv_elems * 4);
  float* dv_acc = reinterpret_cast<float*>(w);
  cudaError_t e = cudaMemsetAsync(dk_acc, 0, kv_elems * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dv_acc, 0, kv_elems * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dk/dv accumulators)");
  FfnBwdPlan fp;
  if ((r = ffn_bwd_plan(attn_out, w_gate, w_up, w_down, dout, p.S, p.h, p.f, p.qb, dw_gate,
                        dw_up, dw_down, ffn_ws, &fp)) != LCA_OK)
    return r;
  const size_t row_q = static_cast<size_t>(p.attn.Hq) * p.attn.d;
  for (int64_t r0 = 0; r0 < p.S; r0 += p.qb) {
    const int rows = static_cast<int>(p.S - r0 < p.qb ? p.S - r0 : p.qb);
    // feedforward backward of the block: its weight gradients, and the
    // gradient of its input rows (the attention output) into dx_blk
    if ((r = ffn_bwd_rows(fp, r0, rows, dx_blk, st)) != LCA_OK) return r;
    // attention backward of the block's query rows with that gradient
    Common c;
    AttnSched s;
    bpt_block(p, causal, r0, rows, &c, &s);
    e = cudaMemcpy2DAsync(lse_blk, rows * sizeof(float), lse + r0, p.S * sizeof(float),
                          rows * sizeof(float), p.attn.Hq, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy2DAsync(lse of a block)");
    const auto* o_rows = static_cast<const __nv_bfloat16*>(attn_out) + r0 * row_q;
    if ((r = bwd_prep(c, o_rows, lse_blk, dx_blk, attn_ws, st)) != LCA_OK) return r;
    if ((r = bwd_main(c, s, static_cast<const __nv_bfloat16*>(q) + r0 * row_q, k, v, dx_blk,
                      attn_ws, nullptr, nullptr, dk_acc, dv_acc, 1, kDefaultBudget, st)) !=
        LCA_OK)
      return r;
    if ((r = bwd_dq(c, attn_ws, static_cast<__nv_bfloat16*>(dq) + r0 * row_q, st)) != LCA_OK)
      return r;
  }
  if ((r = lca_cast_f32_bf16(static_cast<int64_t>(kv_elems), dk_acc, dk, stream)) != LCA_OK)
    return r;
  return lca_cast_f32_bf16(static_cast<int64_t>(kv_elems), dv_acc, dv, stream);
}

lca_status lca_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h[2] = {0, 0};
  e = cudaMemcpyFromSymbol(h, g_err, sizeof h);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (h[0]) {
    const int z[2] = {0, 0};
    cudaMemcpyToSymbol(g_err, z, sizeof z);
    if (h[0] & kErrTimeout)
      return fail(LCA_ERR_TIMEOUT, "a kernel wait ran out (site %d)%s", h[1],
                  (h[0] & kErrDrain) ? "; a CTA then gave up waiting for its work in flight"
                                     : "");
    if (h[0] & kErrDrain)
      return fail(LCA_ERR_TIMEOUT,
                  "a CTA gave up waiting for its own copies or MMAs in flight (site %d)", h[1]);
    if (h[0] & kErrSeqOffsets)
      return fail(LCA_ERR_INVALID_ARG,
                  "cu_seqlens out of order or range, or a sequence longer than max_seqlen "
                  "(site %d); outputs of that call are undefined",
                  h[1]);
    return fail(LCA_ERR_CUDA, "a kernel could not align its shared-memory layout (site %d)",
                h[1]);
  }
  return LCA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc backward
//
// lca_attn_bwd_noalloc: the backward pass for callers that cannot allocate
// device memory.  Its scratch (the float32 D rows and, for bf16, the float32
// dq accumulator) lives in the fixed array below instead of a caller buffer.
// The array is part of this library's device image, so every GPU that loads
// the library holds LCA_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code may not use the array's name as a device address (on the host it
// is only a stand-in); its device address is looked up once per device with
// cudaGetSymbolAddress while that device is current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LCA_NOALLOC_SCRATCH_BYTES];

namespace {

lca_status noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LCA_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(built-in scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return LCA_OK;
}

}  // namespace

extern "C" lca_status lca_attn_bwd_noalloc(const lca_shape* shape, const void* q, const void* k,
                                           const void* v, const void* out, const float* lse,
                                           const void* dout, int causal, void* dq, void* dk,
                                           void* dv, void* stream) {
  Common c;
  lca_status r = check_shape(shape, &c);
  if (r != LCA_OK) return r;
  if ((r = check_ptrs({q, k, v, out, lse, dout, dq, dk, dv})) != LCA_OK) return r;
  AttnSched s;
  if ((r = make_chunk_sched(c, causal, 0, nullptr, &s)) != LCA_OK) return r;
  const size_t need = ws_bytes_of(c);
  if (need > LCA_NOALLOC_SCRATCH_BYTES)
    return fail(LCA_ERR_WORKSPACE,
                "this shape needs %zu bytes of scratch; the built-in scratch of "
                "lca_attn_bwd_noalloc holds %zu (use lca_attn_bwd with a workspace)",
                need, static_cast<size_t>(LCA_NOALLOC_SCRATCH_BYTES));
  void* ws = nullptr;
  if ((r = noalloc_scratch_address(&ws)) != LCA_OK) return r;
  return run_bwd(c, s, q, k, v, out, lse, dout, dq, dk, dv, ws, LCA_NOALLOC_SCRATCH_BYTES,
                 kDefaultBudget, static_cast<cudaStream_t>(stream));
}
