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
 *   pointers aligned to 16 bytes.  The library allocates no device memory.
 *   Its device image holds two pieces of state that outlive a call: one
 *   error word per device (read and cleared by lca_check), and the fixed
 *   scratch array of lca_attn_bwd_noalloc (LCA_NOALLOC_SCRATCH_BYTES per
 *   device, loaded with the library and kept until the process exits).
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
 * Blocks: one step of a sequence-parallel ring.  Each host keeps its block of
 * query rows, the key/value blocks travel from host to host, and every host
 * attends its queries to each key/value block as it arrives, overlapping the
 * transfer of the next block with the computation (Ring Attention with
 * Blockwise Transformers for Near-Infinite Context, Summary and Key points);
 * the per-block partial results combine into the exact answer whatever the
 * order of arrival.  These calls are the per-host steps; the transfer
 * between hosts is the caller's (the package's ring driver uses NCCL).
 *
 * Shape: B batch entries; a query block of Sq rows (q, dout, out, dq
 * [B, Sq, Hq, d]; lse [B, Hq, Sq]) and a key/value block of Sk rows (k, v
 * [B, Sk, Hkv, d]; dk_acc, dv_acc [B, Sk, Hkv, d] float32).  Query row i
 * sits at position q_pos0 + i and key j at k_pos0 + j of one position
 * axis; with `causal`, key j is visible to query i iff
 * k_pos0 + j <= q_pos0 + i.  bf16 only (LCA_ERR_UNSUPPORTED otherwise).
 * When the diagonal crosses the blocks (some but not all keys visible to
 * some query), q_pos0 - k_pos0 must be a multiple of 128 (the tile);
 * blocks wholly before or wholly after each other have no such rule.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t B, Hq, Hkv;
  int64_t Sq;     /* query rows of the block */
  int64_t Sk;     /* key/value rows of the block */
  int64_t d;      /* 128 */
  int32_t dtype;  /* LCA_BF16 */
  float scale;    /* softmax scale; 0 selects 1/sqrt(d) */
} lca_block_shape;

/* lca_attn_fwd_block -- attend the query block to one key/value block and
 * fold the result into a running one:
 *   partial (O_b, lse_b) over the visible keys of this block (a row that
 *   sees none has the empty partial (0, -inf));
 *   accumulate != 0: (o_acc, lse_acc) <- merge((o_acc, lse_acc), (O_b, lse_b))
 *     with lse = M + ln(e^(lse_acc - M) + e^(lse_b - M)), M the larger,
 *     o = e^(lse_acc - lse) o_acc + e^(lse_b - lse) O_b;
 *   accumulate == 0: (o_acc, lse_acc) <- (O_b, lse_b) (the first block).
 * o_acc: [B, Sq, Hq, d] float32, the running output, normalised (NULL is
 * allowed only with accumulate == 0 and out given); lse_acc: [B, Hq, Sq]
 * float32, natural log, in/out.  out (nullable): the merged output rounded
 * to bf16 (after the last block it is the attention output).  Both are
 * caller-owned device buffers; lse_acc/o_acc are read only when
 * accumulating.  A causal block that no query sees adds nothing and
 * launches nothing when accumulating.
 * Errors: as lca_attn_fwd, plus LCA_ERR_INVALID_ARG for negative
 * positions, misaligned diagonal offsets (above), o_acc and out both NULL,
 * or accumulate without o_acc. */
LCA_API lca_status lca_attn_fwd_block(const lca_block_shape* shape, const void* q,
                                      const void* k, const void* v, int causal, int64_t q_pos0,
                                      int64_t k_pos0, int accumulate, float* o_acc,
                                      float* lse_acc, void* out, void* stream);

/* Workspace of the block backward for one query block: D rows and a
 * padded lse copy ([B, Hq, Sq rounded up to 128] float32 each) and a
 * float32 dq accumulator [B, Sq, Hq, d].  0 for an invalid shape. */
LCA_API size_t lca_attn_bwd_block_workspace_size(const lca_block_shape* shape);

/* lca_attn_bwd_block_prep -- start the backward of a query block: zero the
 * workspace's dq accumulator and compute D_i = dout_i . out_i from the
 * block's FINAL out and lse (over every key of the sequence).  Only Sq of
 * the shape is read (Sk may be anything valid). */
LCA_API lca_status lca_attn_bwd_block_prep(const lca_block_shape* shape, const void* out,
                                           const float* lse, const void* dout, void* workspace,
                                           size_t ws_bytes, void* stream);

/* lca_attn_bwd_block -- add one key/value block's share of the gradients
 * of sum(dout * out): P_ij = exp(scale s_ij - lse_i) recomputed with the
 * final lse, dV_j += sum_i P_ij dO_i, dK_j += scale sum_i dS_ij q_i into
 * the block's accumulators, and dQ_i += scale sum_j dS_ij k_j into the
 * workspace (prepared by lca_attn_bwd_block_prep; blocks may come in any
 * order).  Either dk_acc and dv_acc ([B, Sk, Hkv, d] float32: this block's
 * share is ADDED to them when accumulate_kv != 0, else written over them;
 * the ring's accumulators travel with the key/value block) or dk and dv
 * (bf16, overwritten with this block's share alone) are given, the other
 * pair NULL.
 * Errors: as lca_attn_bwd, plus the block rules above, and
 * LCA_ERR_INVALID_ARG unless exactly one pair is given. */
LCA_API lca_status lca_attn_bwd_block(const lca_block_shape* shape, const void* q,
                                      const void* k, const void* v, const void* dout,
                                      int causal, int64_t q_pos0, int64_t k_pos0,
                                      void* workspace, size_t ws_bytes, float* dk_acc,
                                      float* dv_acc, int accumulate_kv, void* dk, void* dv,
                                      void* stream);

/* lca_attn_bwd_block_dq -- finish the query block: dq (bf16, [B, Sq, Hq,
 * d]) from the workspace's accumulator. */
LCA_API lca_status lca_attn_bwd_block_dq(const lca_block_shape* shape, const void* workspace,
                                         size_t ws_bytes, void* dq, void* stream);

/* lca_cast_f32_bf16 -- dst[i] = bf16(src[i]) (round to nearest even) for n
 * elements: turns a running float32 block result (o_acc, dk_acc, dv_acc)
 * into the bf16 output.  Device pointers, 16-byte aligned.  Errors:
 * LCA_ERR_INVALID_ARG for n <= 0 or NULL/misaligned pointers. */
LCA_API lca_status lca_cast_f32_bf16(int64_t n, const float* src, void* dst, void* stream);

/* lca_accumulate_f32 -- dst[i] += src[i] for n float32 elements: folds a
 * ring step's partial key/value gradients into the accumulators that
 * arrived with the block.  Device pointers, 16-byte aligned, not
 * overlapping.  Errors: as lca_cast_f32_bf16. */
LCA_API lca_status lca_accumulate_f32(int64_t n, const float* src, float* dst, void* stream);

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

/* ---------------------------------------------------------------------------
 * Blockwise Transformer sweep: a host "computes attention and feedforward
 * for its query block block by block" (Ring Attention with Blockwise
 * Transformers for Near-Infinite Context, Summary), and the blockwise
 * feedforward keeps the feedforward's intermediate to one block (Key
 * points).  For each block of q_block query rows in turn: the exact
 * attention of those rows over the keys they see (all keys before the
 * block's last row when causal), then the gated-SiLU feedforward
 * (lca_ffn_fwd's unit) of the block's attention output rows, x =
 * attn_out viewed [S, h] with h = Hq * d.  One sequence (B = 1);
 * bf16, d = 128.
 *   q, attn_out: [S, Hq, d]; k, v: [S, Hkv, d]; lse: [Hq, S] float32;
 *   w_gate, w_up: [f, h]; w_down: [h, f]; out: [S, h] bf16.
 * The attention output of the sweep is the input of its feedforward (no
 * output projection, residual or normalisation in between: those are not
 * part of this library).  Errors: LCA_ERR_INVALID_ARG for dimensions <= 0,
 * q_block not a multiple of 128, NULL or misaligned pointers;
 * LCA_ERR_UNSUPPORTED unless d == 128, h % 256 == 0 and f % 128 == 0 (f %
 * 256 == 0 for the backward); LCA_ERR_WORKSPACE for a missing or small
 * workspace.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t S;        /* tokens of the sequence */
  int64_t Hq, Hkv;  /* attention heads; the feedforward width is h = Hq * d */
  int64_t d;        /* head dimension, 128 */
  int64_t f;        /* feedforward width */
  int64_t q_block;  /* query rows per block, a multiple of 128; 0 selects
                       LCA_FFN_BLOCK_DEFAULT */
  float scale;      /* softmax scale; 0 selects 1/sqrt(d) */
} lca_bpt_shape;

/* Workspace of lca_bpt_fwd: the lse and the feedforward intermediate of one
 * block.  0 for an invalid shape. */
LCA_API size_t lca_bpt_fwd_workspace_size(const lca_bpt_shape* shape);
LCA_API lca_status lca_bpt_fwd(const lca_bpt_shape* shape, const void* q, const void* k,
                               const void* v, int causal, const void* w_gate, const void* w_up,
                               const void* w_down, void* attn_out, float* lse, void* out,
                               void* workspace, size_t ws_bytes, void* stream);

/* lca_bpt_bwd -- gradients of sum(dout * out) of lca_bpt_fwd, block by
 * block: the feedforward backward of the block's rows (weight gradients
 * ADDED to the float32 dw_gate, dw_up, dw_down, as lca_ffn_bwd), whose input
 * gradient is the dout of the block's attention rows; their attention
 * backward recomputes P from lse (dq of the block's rows; dk, dv over every
 * block are summed in float32 inside the workspace and written as bf16 at
 * the end).  attn_out and lse are lca_bpt_fwd's.  dq: [S, Hq, d]; dk, dv:
 * [S, Hkv, d], bf16, overwritten. */
LCA_API size_t lca_bpt_bwd_workspace_size(const lca_bpt_shape* shape);
LCA_API lca_status lca_bpt_bwd(const lca_bpt_shape* shape, const void* q, const void* k,
                               const void* v, int causal, const void* w_gate, const void* w_up,
                               const void* w_down, const void* attn_out, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, float* dw_gate,
                               float* dw_up, float* dw_down, void* workspace, size_t ws_bytes,
                               void* stream);

/* Synchronises `stream`, then reports and clears the device error word of
 * the current device: LCA_ERR_TIMEOUT if a kernel wait ran out since the
 * last check, or if a CTA gave up waiting (about one second) for its own
 * copies or MMAs in flight before it freed its tensor memory (the detail
 * text of lca_last_error says which); LCA_ERR_INVALID_ARG if a kernel met
 * invalid packed sequence offsets, LCA_ERR_CUDA if the stream holds a CUDA
 * error, else LCA_OK. */
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
