// sched.cuh -- which key/value tiles a query tile visits, and in what order.
//
// Positions vs tokens.  Tiles are walked in POSITION space.  For ordinary
// attention a position is a token.  For LongLoRA's S2-Attn (LongLoRA,
// Summary: attention inside groups, half the heads shifted by half a group)
// a shifted head sees position p holding token (p + G/2) mod S; the tile
// walk stays inside the query's group and each position tile maps to one
// contiguous token tile because G/2 is a whole number of tiles.
//
// Ragged lengths: when S is not a multiple of the tile, the last tile is
// partial and the last chunk may hold fewer tiles.
//
// Chunk order (Ring Attention with Blockwise Transformers, Summary: a query
// block meets the key/value blocks in the order the ring delivers them, and
// the result does not depend on it).  Keys are split into chunks of
// `tiles_per_chunk` tiles; a query tile visits the chunks in order
// (in-order), ring order (query block i: chunks i, i-1, ..., i+1 mod n) or a
// caller-given permutation, and the tiles inside a chunk in ascending order.
// Causal chunks/tiles after the query tile are skipped.
#pragma once

#include <stdint.h>

#include "../../include/lca.h"

namespace lca {

struct AttnSched {
  int S;                   // sequence length in tokens
  int n_tiles;             // ceil(S / tile); the last tile may be partial
  int causal;
  int s2;                  // 1: S2-Attn walk
  int tiles_per_chunk;     // chunked walk
  int n_chunks;
  int order;               // lca_order
  int q_block_tiles;       // ring query block, in tiles
  int group_tiles;         // S2: group / tile
  int shift_tiles;         // S2: (group / 2) / tile
  int first_shifted_head;  // S2: Hq - shift_heads
  uint16_t perm[LCA_MAX_CHUNKS];
};

__host__ __device__ inline bool head_shifted(const AttnSched& s, int h) {
  return s.s2 && h >= s.first_shifted_head;
}

// Token tile held by position tile t.
__host__ __device__ inline int token_tile(const AttnSched& s, int t, bool shifted) {
  return shifted ? (t + s.shift_tiles) % s.n_tiles : t;
}

// Walk of the key/value position tiles for query position tile qt.
struct KvWalk {
  const AttnSched* s;
  int qt, ci, t, t_end, qb;

  __host__ __device__ void init(const AttnSched* sc, int qt_) {
    s = sc;
    qt = qt_;
    ci = 0;
    if (s->s2) {
      const int g0 = (qt / s->group_tiles) * s->group_tiles;
      t = g0;
      t_end = s->causal ? qt + 1 : g0 + s->group_tiles;
    } else {
      t = t_end = 0;
      qb = qt / s->q_block_tiles;
    }
  }
  __host__ __device__ int chunk_at(int i) const {
    if (s->order == LCA_ORDER_RING) {
      const int n = s->n_chunks;
      return ((qb - i) % n + n) % n;
    }
    if (s->order == LCA_ORDER_CUSTOM) return s->perm[i];
    return i;
  }
  // Next key/value position tile; false when the walk is over.
  __host__ __device__ bool next(int& tile) {
    if (s->s2) {
      if (t < t_end) {
        tile = t++;
        return true;
      }
      return false;
    }
    while (t >= t_end) {
      if (ci >= s->n_chunks) return false;
      const int c = chunk_at(ci++);
      t = c * s->tiles_per_chunk;
      t_end = t + s->tiles_per_chunk;
      if (t_end > s->n_tiles) t_end = s->n_tiles;  // last chunk may be partial
      if (s->causal && t_end > qt + 1) t_end = qt + 1;
    }
    tile = t++;
    return true;
  }
};

// Query position tiles whose walk contains key position tile kt (for the
// backward pass, which loops over queries for a fixed key tile).
struct QWalk {
  int t, t_end;
  __host__ __device__ void init(const AttnSched* s, int kt) {
    if (s->s2) {
      const int g0 = (kt / s->group_tiles) * s->group_tiles;
      t = s->causal ? kt : g0;
      t_end = g0 + s->group_tiles;
    } else {
      t = s->causal ? kt : 0;
      t_end = s->n_tiles;
    }
  }
  __host__ __device__ int count() const { return t_end - t; }
};

}  // namespace lca
