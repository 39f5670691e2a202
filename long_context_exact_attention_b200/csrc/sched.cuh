// sched.cuh -- which key/value tiles a query tile visits, and in what order.
//
// Positions vs tokens.  Tiles are walked in POSITION space.  For ordinary
// attention a position is a token.  For LongLoRA's S2-Attn (LongLoRA,
// Summary: attention inside groups, half the heads shifted by half a group)
// a shifted head sees position p holding token (p + G/2) mod S; the tile
// walk stays inside the query's group and each position tile maps to one
// contiguous token tile because G/2 is a whole number of tiles.
//
// Sequences.  A batch entry is one sequence of S tokens, or -- for packed
// variable-length batches -- sequence b holds tokens [cu[b], cu[b+1]) of one
// packed token axis.  Every walk runs inside one sequence, with positions
// counted from its first token.  When a sequence's length is not a multiple
// of the tile its last tile is partial.
//
// Blocks.  A sequence-parallel caller attends a block of queries to a block
// of keys that starts elsewhere on the position axis (Ring Attention with
// Blockwise Transformers, Summary: each host keeps its query block and sees
// the key/value blocks of the others in turn).  Then the key block has its
// own length S_kv and the causal diagonal is shifted: key tile T is on the
// diagonal of query tile Q when T == Q + diag (diag = (query position -
// key position of the blocks' first rows) / tile), visible in full before
// it and invisible after it.  Ordinary calls have S_kv == S and diag == 0.
//
// Chunk order (Ring Attention with Blockwise Transformers, Summary: a query
// block meets the key/value blocks in the order the ring delivers them, and
// the result does not depend on it).  Keys are split into chunks of
// `kv_chunk` keys, any length; a query tile visits the chunks in order
// (in-order), ring order (query block i: chunks i, i-1, ..., i+1 mod n) or a
// caller-given permutation, and the tiles inside a chunk in ascending order.
// A tile that straddles a chunk boundary is visited once per chunk, each
// visit restricted to that chunk's keys [lo, hi).  Causal tiles after the
// query tile are skipped.
#pragma once

#include <stdint.h>

#include "../../include/lca.h"

namespace lca {

struct AttnSched {
  int S;                   // longest sequence in tokens (every sequence when not packed)
  int n_tiles;             // ceil(S / tile)
  int S_kv;                // keys of a dense sequence (== S except for block calls)
  int n_kv_tiles;          // ceil(S_kv / tile)
  int diag;                // causal: key tile Q + diag is the diagonal of query tile Q
  int tile;                // tokens per tile
  int causal;
  int s2;                  // 1: S2-Attn walk
  int kv_chunk;            // chunked walk: keys per chunk (>= 1)
  int n_chunks;            // chunks of a sequence of S tokens
  int order;               // lca_order
  int q_block;             // ring query block, in tokens
  int group_tiles;         // S2: group / tile
  int shift_tiles;         // S2: (group / 2) / tile
  int first_shifted_head;  // S2: Hq - shift_heads
  const int* cu_seqlens;   // packed sequences: n_seqs + 1 token offsets (device), else null
  uint16_t perm[LCA_MAX_CHUNKS];
};

__host__ __device__ inline bool head_shifted(const AttnSched& s, int h) {
  return s.s2 && h >= s.first_shifted_head;
}

// Token tile held by position tile t.
__host__ __device__ inline int token_tile(const AttnSched& s, int t, bool shifted) {
  return shifted ? (t + s.shift_tiles) % s.n_tiles : t;
}

// Where sequence b lives in the tensors: tensor coordinates (batch index bm,
// first token tokb), its first row on the flattened token axis of all batch
// entries (row0 = bm * S_tensor + tokb) and its length; the same for its
// keys (kv_row0, kv_len), which differ only for block calls.  S_tensor is
// the token extent of one batch entry of the query tensors (the packed
// length for packed sequences); a dense key tensor holds S_kv tokens per
// batch entry.
struct SeqView {
  int bm, tokb, row0, len, n_tiles;
  int kv_row0, kv_len, kv_n_tiles;
};

// False when packed offsets are out of order or out of range (the caller
// records an error and does no work for the sequence).
__host__ __device__ inline bool seq_view(const AttnSched& s, int b, int S_tensor, SeqView* v) {
  if (!s.cu_seqlens) {
    v->bm = b;
    v->tokb = 0;
    v->row0 = b * S_tensor;
    v->len = s.S;
    v->n_tiles = s.n_tiles;
    v->kv_row0 = b * s.S_kv;
    v->kv_len = s.S_kv;
    v->kv_n_tiles = s.n_kv_tiles;
    return true;
  }
  const int c0 = s.cu_seqlens[b], c1 = s.cu_seqlens[b + 1];
  if (c0 < 0 || c1 < c0 || c1 > S_tensor || c1 - c0 > s.S) return false;
  v->bm = 0;
  v->tokb = c0;
  v->row0 = c0;
  v->len = c1 - c0;
  v->n_tiles = (v->len + s.tile - 1) / s.tile;
  v->kv_row0 = v->row0;
  v->kv_len = v->len;
  v->kv_n_tiles = v->n_tiles;
  return true;
}

// Walk of the key/value position tiles for query position tile qt of a
// sequence whose keys number `len`.
struct KvWalk {
  const AttnSched* s;
  int qt, len, n_chunks, key_end;
  int ci, t, t_end, c_lo, c_hi, qb;

  __host__ __device__ void init(const AttnSched* sc, int qt_, int len_) {
    s = sc;
    qt = qt_;
    len = len_;
    ci = 0;
    if (s->s2) {
      const int g0 = (qt / s->group_tiles) * s->group_tiles;
      t = g0;
      t_end = s->causal ? qt + 1 : g0 + s->group_tiles;
    } else {
      t = t_end = 0;
      n_chunks = (len + s->kv_chunk - 1) / s->kv_chunk;
      // keys past the query tile's last row are invisible under the mask
      key_end = len;
      if (s->causal && (qt + 1 + s->diag) * s->tile < key_end)
        key_end = (qt + 1 + s->diag) * s->tile;
      qb = qt * s->tile / s->q_block;
    }
  }
  __host__ __device__ int chunk_at(int i) const {
    if (s->order == LCA_ORDER_RING) {
      const int n = n_chunks;
      return ((qb - i) % n + n) % n;
    }
    if (s->order == LCA_ORDER_CUSTOM) return s->perm[i];
    return i;
  }
  // Next visit: key/value position tile and the key range [lo, hi) of it
  // (offsets inside the tile) that the visit covers; false when the walk is
  // over.
  __host__ __device__ bool next(int& tile, int& lo, int& hi) {
    if (s->s2) {
      if (t < t_end) {
        tile = t++;
        lo = 0;
        hi = s->tile;
        return true;
      }
      return false;
    }
    while (t >= t_end) {
      if (ci >= n_chunks) return false;
      const int c = chunk_at(ci++);
      c_lo = c * s->kv_chunk;
      c_hi = c_lo + s->kv_chunk;
      if (c_hi > key_end) c_hi = key_end;
      if (c_lo >= c_hi) continue;  // nothing visible in this chunk
      t = c_lo / s->tile;
      t_end = (c_hi - 1) / s->tile + 1;
    }
    tile = t++;
    const int k0 = tile * s->tile;
    lo = c_lo > k0 ? c_lo - k0 : 0;
    hi = c_hi - k0 < s->tile ? c_hi - k0 : s->tile;
    return true;
  }
};

// The same walk when every chunk is a whole number of tiles: no visit is
// split, so it yields tiles only (the forward kernel's fast path; a ragged
// last tile is masked there from the sequence length).  Visits the same
// tiles in the same order as KvWalk for such chunks.
struct TileWalk {
  const AttnSched* s;
  int qt, n_tiles, tpc, n_chunks, ci, t, t_end, qb;

  __host__ __device__ void init(const AttnSched* sc, int qt_, int n_tiles_) {
    s = sc;
    qt = qt_;
    n_tiles = n_tiles_;
    ci = 0;
    if (s->s2) {
      const int g0 = (qt / s->group_tiles) * s->group_tiles;
      t = g0;
      t_end = s->causal ? qt + 1 : g0 + s->group_tiles;
    } else {
      t = t_end = 0;
      tpc = s->kv_chunk / s->tile;
      n_chunks = (n_tiles + tpc - 1) / tpc;
      qb = qt * s->tile / s->q_block;
    }
  }
  __host__ __device__ int chunk_at(int i) const {
    if (s->order == LCA_ORDER_RING) {
      const int n = n_chunks;
      return ((qb - i) % n + n) % n;
    }
    if (s->order == LCA_ORDER_CUSTOM) return s->perm[i];
    return i;
  }
  __host__ __device__ bool next(int& tile) {
    if (s->s2) {
      if (t < t_end) {
        tile = t++;
        return true;
      }
      return false;
    }
    while (t >= t_end) {
      if (ci >= n_chunks) return false;
      const int c = chunk_at(ci++);
      t = c * tpc;
      t_end = t + tpc;
      if (t_end > n_tiles) t_end = n_tiles;
      if (s->causal && t_end > qt + 1 + s->diag) t_end = qt + 1 + s->diag;
    }
    tile = t++;
    return true;
  }
};

// Query position tiles whose walk contains key position tile kt, for a
// sequence of n_tiles query tiles (the backward pass loops over queries for
// a fixed key tile).
struct QWalk {
  int t, t_end;
  __host__ __device__ void init(const AttnSched* s, int kt, int n_tiles) {
    if (s->s2) {
      const int g0 = (kt / s->group_tiles) * s->group_tiles;
      t = s->causal ? kt : g0;
      t_end = g0 + s->group_tiles;
    } else {
      t = (s->causal && kt - s->diag > 0) ? kt - s->diag : 0;
      t_end = n_tiles;
    }
  }
  __host__ __device__ int count() const { return t_end > t ? t_end - t : 0; }
};

}  // namespace lca
