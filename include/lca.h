/*
 * lca.h -- exact long-context attention on NVIDIA B200 (sm_100a): C ABI.
 *
 * What it computes
 *   Exact softmax attention, softmax(Q K^T * scale + mask) V, together with
 *   the per-row log-sum-exp (lse) and the gradients that recompute the
 *   attention matrix from that lse.  "Attention stays exact" while it is
 *   computed block by block, and the per-block partial results combine to
 *   the same answer whatever order the key/value blocks arrive in (Ring
 *   Attention with Blockwise Transformers for Near-Infinite Context,
 *   Summary).  Full attention with no approximation is what the 700K/1M
 *   token recipes train with (sourcepulse project card of the 1M-context
 *   training recipe, How It Works).  LongLoRA's shifted sparse attention
 *   (LongLoRA: Efficient Fine-tuning of Long-Context Large Language Models,
 *   Summary) is the same computation restricted to groups, with half the
 *   heads shifted by half a group.
 *
 * Layouts (all tensors dense, row-major, no padding)
 *   q, out, dout, dq : [B, S, Hq,  d]   (token-major, head dim contiguous)
 *   k, v, dk, dv     : [B, S, Hkv, d]
 *   lse              : [B, Hq, S] float32, natural log of sum_j exp(scale*s_ij)
 *   Grouped-query heads: query head h reads key/value head h / (Hq / Hkv).
 *   Causal: key j is visible to query i iff j <= i (one position axis).
 *
 * Element types
 *   LCA_BF16: q, k, v, out, dout, dq, dk, dv are bfloat16; accumulation in
 *             float32 on the tensor cores; requires d == 128; tiles of 128.
 *   LCA_FP32: every tensor float32, exact float32 arithmetic on CUDA cores;
 *             d in {64, 128}; tiles of 64.
 *   Any S >= 1: when S is not a multiple of the tile the last tile is
 *   partial (ragged); S2-Attn needs S to be a multiple of its group.
 *
 * Ownership and memory
 *   The caller allocates every device buffer (inputs, outputs, workspace)
 *   and keeps it alive until the stream work completes.  Pointers are device
 *   pointers aligned to 16 bytes.  The library allocates no device memory;
 *   it keeps no state between calls except one device error word per device.
 *
 * Errors
 *   Argument errors are returned synchronously, before anything is launched.
 *   A failed launch returns LCA_ERR_CUDA.  Every kernel bounds each of its
 *   waits; a wait that runs out sets the device error word and the kernel
 *   returns early (its outputs are then undefined).  lca_check() reports it.
 *   Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and thread-safe.
 */
#ifndef LCA_H
#define LCA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LCA_API __attribute__((visibility("default")))
#else
#define LCA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LCA_OK = 0,
  LCA_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or option     */
  LCA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. bf16 d=64)  */
  LCA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed           */
  LCA_ERR_TIMEOUT = 4,      /* a kernel wait ran out (see lca_check)       */
  LCA_ERR_WORKSPACE = 5     /* workspace missing or smaller than required  */
} lca_status;

typedef enum { LCA_BF16 = 0, LCA_FP32 = 1 } lca_dtype;

/* Order in which a query tile visits the key/value chunks.  The result does
 * not depend on it beyond float32 rounding (Ring Attention, Summary). */
typedef enum {
  LCA_ORDER_INORDER = 0, /* chunks 0, 1, ..., n-1                              */
  LCA_ORDER_RING = 1,    /* query block i visits chunks i, i-1, ..., i+1 (mod n),
                            the order in which a ring delivers them            */
  LCA_ORDER_CUSTOM = 2   /* opts->chunk_perm[0..n-1], a permutation of 0..n-1  */
} lca_order;

typedef struct {
  int64_t B, Hq, Hkv, S, d;
  int32_t dtype;  /* lca_dtype */
  float scale;    /* softmax scale; 0 selects 1/sqrt(d) */
} lca_shape;

typedef struct {
  int32_t order;              /* lca_order                                   */
  const int32_t* chunk_perm;  /* HOST array of n_chunks entries (CUSTOM only) */
  int64_t q_block;            /* RING: query-block length in tokens, 0 =
                                 kv_chunk.  A query tile follows the ring
                                 position of the block holding its first row;
                                 the bf16 path walks two query tiles together,
                                 in the order of the second.                 */
  uint64_t timeout_cycles;    /* per-wait budget in SM clocks; 0 = default
                                 (2^31, about one second)                    */
} lca_opts;

#define LCA_MAX_CHUNKS 1024

/* ---------------------------------------------------------------------------
 * lca_attn_fwd -- exact attention forward over key/value chunks.
 *   The keys are split into ceil(S / kv_chunk) chunks of kv_chunk keys
 *   (kv_chunk == 0 or >= S: one chunk; the last chunk may be partial).
 *   kv_chunk need not be a multiple of the tile: a key tile that straddles
 *   a chunk boundary is visited once per chunk, each visit masked to that
 *   chunk's keys.
 *   Each query tile attends to the chunks in the order opts selects; the
 *   partial (O, lse) of every chunk is folded into the running result in
 *   unnormalised form (running max m, running sum l, running O*l), which is
 *   the log-sum-exp merge of the Ring Attention summary carried out chunk by
 *   chunk.  Causal chunks/tiles that hold no visible key are skipped.
 *   q, k, v: inputs (layouts above).  out: [B,S,Hq,d] output, same dtype.
 *   lse: [B,Hq,S] float32 output.  opts may be NULL (in-order).
 *   Errors: LCA_ERR_INVALID_ARG when a pointer is NULL or misaligned, a
 *   dimension is <= 0, Hq % Hkv != 0, kv_chunk or q_block is negative,
 *   the chunk count exceeds LCA_MAX_CHUNKS, or the
 *   permutation is invalid; LCA_ERR_UNSUPPORTED for shapes outside the
 *   element-type limits above.
 * ------------------------------------------------------------------------- */
LCA_API lca_status lca_attn_fwd(const lca_shape* shape, const void* q, const void* k,
                        const void* v, int causal, int64_t kv_chunk,
                        const lca_opts* opts, void* out, float* lse,
                        void* stream);

/* Bytes of device workspace lca_attn_bwd / lca_s2attn_bwd need: float32
 * rows D_i = dout_i . out_i and a copy of lse, each [B,Hq,S rounded up to
 * the tile], and, for bf16, a float32 dq accumulator ([B,S,Hq,d]).  Returns
 * 0 for an invalid shape. */
LCA_API size_t lca_attn_bwd_workspace_size(const lca_shape* shape);

/* ---------------------------------------------------------------------------
 * lca_attn_bwd -- gradients of sum(dout * out) with respect to q, k, v.
 *   P is recomputed from q, k and the saved lse (no attention matrix is
 *   stored): P_ij = exp(scale*s_ij - lse_i), dV = P^T dO, dP = dO V^T,
 *   dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q, D_i = dO_i . O_i.
 *   With grouped-query heads dk/dv sum over the query heads of a group.
 *   out and lse must come from lca_attn_fwd on the same inputs and `causal`.
 *   dq, dk, dv: outputs, input dtype, fully overwritten.  workspace: device
 *   buffer of ws_bytes >= lca_attn_bwd_workspace_size(shape) bytes, owned
 *   by the caller, contents need not be initialised.
 *   Errors: as lca_attn_fwd; LCA_ERR_WORKSPACE when the workspace is NULL
 *   or too small.
 * ------------------------------------------------------------------------- */
LCA_API lca_status lca_attn_bwd(const lca_shape* shape, const void* q, const void* k,
                        const void* v, const void* out, const float* lse,
                        const void* dout, int causal, void* dq, void* dk,
                        void* dv, void* workspace, size_t ws_bytes,
                        void* stream);

/* ---------------------------------------------------------------------------
 * lca_attn_bwd_noalloc -- lca_attn_bwd for callers that cannot allocate
 * device memory.  No counterpart in the pages: it exists for callers such
 * as a plugin inside a host framework that owns every device allocation and
 * hands the plugin none, or code on a latency-critical path that cannot take
 * cudaMalloc's cost and implicit synchronisation.  The caller still passes
 * every input and output; the scratch that lca_attn_bwd takes as
 * `workspace` (float32 D rows and, for bf16, a float32 dq accumulator:
 * lca_attn_bwd_workspace_size bytes) comes instead from a fixed array of
 * LCA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  The function allocates and
 * frees nothing.
 *   Set-up: the first call on each device looks up the array's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture.
 *   Sharing: every call on a device uses the same array and leaves its last
 *   contents there (the parts that must start at zero are cleared by each
 *   call).  Calls whose work overlaps on the GPU -- on different streams, or
 *   from different host threads without ordering -- race on the array and
 *   give wrong gradients; issue them in order, e.g. on one stream.
 *   Errors: as lca_attn_bwd; LCA_ERR_WORKSPACE when the shape needs more
 *   scratch than LCA_NOALLOC_SCRATCH_BYTES (use lca_attn_bwd then).
 * ------------------------------------------------------------------------- */
#define LCA_NOALLOC_SCRATCH_BYTES (64u << 20)
LCA_API lca_status lca_attn_bwd_noalloc(const lca_shape* shape, const void* q,
                                        const void* k, const void* v,
                                        const void* out, const float* lse,
                                        const void* dout, int causal, void* dq,
                                        void* dk, void* dv, void* stream);

/* ---------------------------------------------------------------------------
 * lca_s2attn_fwd -- LongLoRA shifted sparse attention (S2-Attn), forward.
 *   Positions are split into S/group groups of `group`; attention runs
 *   inside each group (causal by position within the group when `causal`).
 *   The trailing `shift_heads` query heads (and the key/value heads they
 *   read) are shifted by group/2: shifted position p holds original token
 *   (p + group/2) mod S, so the last group wraps around.  Outputs and lse
 *   are in ORIGINAL token order; the shift is applied to tile coordinates
 *   inside the kernel, no tensor is rolled.  shift_heads == 0 gives the
 *   unshifted short attention; group == S with shift_heads == 0 is full
 *   attention.
 *   When group/2 is a whole number of tiles (128 bf16, 64 fp32) the shift
 *   lives in the kernels' tile coordinates and no workspace is needed.
 *   Other even groups (LongLoRA's 100K context: S = 100000, group 25000)
 *   need lca_s2attn_fwd_ws: the heads are rolled into its workspace, the
 *   groups run as a packed batch, and the results are rolled back.
 *   Errors: as lca_attn_fwd, plus LCA_ERR_INVALID_ARG when group is odd or
 *   does not divide S, shift_heads is outside [0, Hq], or the shifted heads
 *   do not cover whole grouped-query groups; LCA_ERR_WORKSPACE from
 *   lca_s2attn_fwd for a group that needs a workspace.
 * ------------------------------------------------------------------------- */
LCA_API lca_status lca_s2attn_fwd(const lca_shape* shape, const void* q, const void* k,
                          const void* v, int causal, int64_t group,
                          int64_t shift_heads, void* out, float* lse,
                          void* stream);

/* lca_s2attn_fwd_ws -- lca_s2attn_fwd with a workspace of at least
 * lca_s2attn_fwd_workspace_size bytes (0 for groups whose half is a whole
 * number of tiles, then workspace may be NULL). */
LCA_API size_t lca_s2attn_fwd_workspace_size(const lca_shape* shape, int64_t group,
                                             int64_t shift_heads);
LCA_API lca_status lca_s2attn_fwd_ws(const lca_shape* shape, const void* q, const void* k,
                                     const void* v, int causal, int64_t group,
                                     int64_t shift_heads, void* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream);

/* lca_s2attn_bwd -- gradients of S2-Attn; arguments as lca_attn_bwd plus
 * group/shift_heads as lca_s2attn_fwd.  The workspace must hold
 * lca_s2attn_bwd_workspace_size bytes (lca_attn_bwd_workspace_size when
 * group/2 is a whole number of tiles; more otherwise, for the rolled
 * tensors). */
LCA_API size_t lca_s2attn_bwd_workspace_size(const lca_shape* shape, int64_t group,
                                             int64_t shift_heads);
LCA_API lca_status lca_s2attn_bwd(const lca_shape* shape, const void* q, const void* k,
                          const void* v, const void* out, const float* lse,
                          const void* dout, int causal, int64_t group,
                          int64_t shift_heads, void* dq, void* dk, void* dv,
                          void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Packed variable-length batches.  No counterpart in the pages, which train
 * on fixed-length sequences; callers that pack documents of different
 * lengths into one token axis need it ("nearly 1M"-token contexts are not a
 * multiple of any tile either).
 *   shape->B is the number of sequences n and shape->S the total number of
 *   packed tokens T.  Sequence b holds tokens [cu_seqlens[b], cu_seqlens[b+1])
 *   and attends only to itself (causal by position inside the sequence);
 *   cu_seqlens is a DEVICE array of n + 1 int32 offsets, nondecreasing, from
 *   0 up to at most T, and no sequence is longer than max_seqlen (which sets
 *   the grid and the workspace).  Empty sequences are allowed.
 *   Layouts: q, out, dout, dq [T, Hq, d]; k, v, dk, dv [T, Hkv, d];
 *   lse [Hq, T] float32.  Token rows outside every sequence are left
 *   untouched in out, lse, dk and dv and are set to zero in dq.  The last
 *   tile of a sequence reads the rows that follow it (the next sequence, or
 *   rows outside every sequence) and multiplies them by zero, so every row
 *   of q, k, v and dout below T must hold finite values.
 *   Chunking and chunk order apply inside each sequence; LCA_ORDER_CUSTOM is
 *   rejected (sequences have different chunk counts).
 *   Errors: as the dense calls, plus LCA_ERR_INVALID_ARG for a NULL or
 *   misaligned cu_seqlens or max_seqlen outside [1, T].  Offsets that are
 *   out of order, out of range or longer than max_seqlen cannot be checked
 *   before launch (they live on the device): the kernels skip the affected
 *   sequence and lca_check() then returns LCA_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------- */
LCA_API lca_status lca_attn_fwd_varlen(const lca_shape* shape, const int32_t* cu_seqlens,
                                       int64_t max_seqlen, const void* q, const void* k,
                                       const void* v, int causal, int64_t kv_chunk,
                                       const lca_opts* opts, void* out, float* lse,
                                       void* stream);

/* Workspace bytes of lca_attn_bwd_varlen: D rows and a copy of lse, each
 * [n, Hq, max_seqlen rounded up to the tile] float32, and, for bf16, a
 * float32 dq accumulator [T, Hq, d].  0 for an invalid shape. */
LCA_API size_t lca_attn_bwd_varlen_workspace_size(const lca_shape* shape, int64_t max_seqlen);

LCA_API lca_status lca_attn_bwd_varlen(const lca_shape* shape, const int32_t* cu_seqlens,
                                       int64_t max_seqlen, const void* q, const void* k,
                                       const void* v, const void* out, const float* lse,
                                       const void* dout, int causal, void* dq, void* dk,
                                       void* dv, void* workspace, size_t ws_bytes,
                                       void* stream);

/* ---------------------------------------------------------------------------
 * lca_lse_merge -- combine two partial attention results over disjoint key
 * sets (Ring Attention, Summary: per-block results combine independently of
 * order):  lse = M + ln(e^(lse_a-M) + e^(lse_b-M)), M = max(lse_a, lse_b);
 * o = e^(lse_a-lse) o_a + e^(lse_b-lse) o_b.  A row with lse = -inf is an
 * empty partial (identity).  o_*: [rows, d] float32, lse_*: [rows] float32,
 * all device pointers; o_out/lse_out may alias o_a/lse_a.
 * Errors: LCA_ERR_INVALID_ARG for rows/d <= 0 or NULL pointers.
 * ------------------------------------------------------------------------- */
LCA_API lca_status lca_lse_merge(int64_t rows, int64_t d, const float* o_a,
                         const float* lse_a, const float* o_b,
                         const float* lse_b, float* o_out, float* lse_out,
                         void* stream);

/* ---------------------------------------------------------------------------
 * Blockwise feedforward.  A host of the ring computes attention and the
 * feedforward for its query block block by block, and the blockwise
 * feedforward is what lowers the feedforward's activation memory (Ring
 * Attention with Blockwise Transformers for Near-Infinite Context, Summary
 * and Key points).  The pages print no feedforward; this is Llama's gated
 * SiLU unit, with PyTorch's Linear weight layout:
 *     H   = silu(x W_gate^T) * (x W_up^T),   silu(g) = g / (1 + e^-g)
 *     out = H W_down^T
 * x, out: [T, h] bf16; w_gate, w_up: [f, h] bf16; w_down: [h, f] bf16.
 * The token rows are processed block_tokens at a time (0 selects
 * LCA_FFN_BLOCK_DEFAULT; capped at T rounded up to 128), so the
 * intermediate H exists for one block only: it lives in the caller's
 * workspace of block_tokens * f bf16 (lca_ffn_workspace_size).  Products
 * accumulate in float32 on the tensor cores; H is rounded to bf16.
 * Errors: LCA_ERR_INVALID_ARG for dimensions <= 0, a block_tokens that is
 * negative or not a multiple of 128, NULL or misaligned pointers;
 * LCA_ERR_UNSUPPORTED unless h % 256 == 0 and f % 128 == 0 (every Llama
 * size); LCA_ERR_WORKSPACE when the workspace is NULL or too small.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t T;  /* token rows */
  int64_t h;  /* model width */
  int64_t f;  /* feedforward width */
} lca_ffn_shape;

#define LCA_FFN_BLOCK_DEFAULT 8192

LCA_API size_t lca_ffn_workspace_size(const lca_ffn_shape* shape, int64_t block_tokens);

LCA_API lca_status lca_ffn_fwd(const lca_ffn_shape* shape, const void* x, const void* w_gate,
                               const void* w_up, const void* w_down, int64_t block_tokens,
                               void* out, void* workspace, size_t ws_bytes, void* stream);

/* lca_ffn_bwd -- gradients of sum(dout * out) of lca_ffn_fwd, block by
 * block with the gate and up products recomputed from x:
 *     dH = dout W_down;   dU = dH * silu(G);   dG = dH * U * silu'(G)
 *     dx = dG W_gate + dU W_up
 *     dw_gate += dG^T x;  dw_up += dU^T x;  dw_down += dout^T H
 * dout: [T, h] bf16; dx: [T, h] bf16, overwritten; dw_gate, dw_up [f, h]
 * and dw_down [h, f] are FLOAT32 and the gradients are ADDED to them (zero
 * them first for a fresh gradient).  workspace: lca_ffn_bwd_workspace_size
 * bytes (dH, dG, dU and H of one block, bf16).  Errors: as lca_ffn_fwd, and
 * LCA_ERR_UNSUPPORTED unless f % 256 == 0. */
LCA_API size_t lca_ffn_bwd_workspace_size(const lca_ffn_shape* shape, int64_t block_tokens);

LCA_API lca_status lca_ffn_bwd(const lca_ffn_shape* shape, const void* x, const void* w_gate,
                               const void* w_up, const void* w_down, const void* dout,
                               int64_t block_tokens, void* dx, float* dw_gate, float* dw_up,
                               float* dw_down, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reports and clears the device error word of
 * the current device: LCA_ERR_TIMEOUT if a kernel wait ran out since the
 * last check, LCA_ERR_INVALID_ARG if a kernel met invalid packed sequence
 * offsets, LCA_ERR_CUDA if the stream holds a CUDA error, else LCA_OK. */
LCA_API lca_status lca_check(void* stream);

/* Static description of a status code. */
LCA_API const char* lca_status_string(lca_status s);

/* Human-readable detail of the last non-OK status returned on this host
 * thread (which argument, which CUDA error).  Never NULL. */
LCA_API const char* lca_last_error(void);

/* Library version, (major << 16) | minor. */
LCA_API int lca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LCA_H */
