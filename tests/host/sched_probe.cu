// Host-side probe of the tile walks in sched.cuh: prints, for the schedule
// given on the command line, every query tile's visits (key tile and the
// key range [lo, hi) inside it), the tile-only walk's tiles when chunks are
// whole tiles, every key tile's query tile range, and the position -> token
// tile map.  Built and run by tests/test_sched_host.py.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../long_context_exact_attention_b200/csrc/sched.cuh"

int main(int argc, char** argv) {
  // args: S tile causal s2 kv_chunk order q_block group_tiles shift_tiles
  //       first_shifted_head [perm...]
  if (argc < 11) return 2;
  lca::AttnSched s;
  std::memset(&s, 0, sizeof s);
  s.S = atoi(argv[1]);
  s.tile = atoi(argv[2]);
  s.n_tiles = (s.S + s.tile - 1) / s.tile;
  s.causal = atoi(argv[3]);
  s.s2 = atoi(argv[4]);
  s.kv_chunk = atoi(argv[5]);
  s.n_chunks = s.kv_chunk ? (s.S + s.kv_chunk - 1) / s.kv_chunk : 1;
  s.order = atoi(argv[6]);
  s.q_block = atoi(argv[7]);
  s.group_tiles = atoi(argv[8]);
  s.shift_tiles = atoi(argv[9]);
  s.first_shifted_head = atoi(argv[10]);
  for (int i = 11; i < argc && i - 11 < LCA_MAX_CHUNKS; ++i) s.perm[i - 11] = atoi(argv[i]);
  for (int qt = 0; qt < s.n_tiles; ++qt) {
    lca::KvWalk w;
    w.init(&s, qt, s.S);
    printf("Q %d:", qt);
    int t, lo, hi;
    while (w.next(t, lo, hi)) printf(" %d,%d,%d", t, lo, hi);
    printf("\n");
  }
  // the tile-only walk, for chunks of whole tiles (S2 included)
  if (s.s2 || s.kv_chunk % s.tile == 0) {
    for (int qt = 0; qt < s.n_tiles; ++qt) {
      lca::TileWalk w;
      w.init(&s, qt, s.n_tiles);
      printf("W %d:", qt);
      int t;
      while (w.next(t)) printf(" %d", t);
      printf("\n");
    }
  }
  for (int kt = 0; kt < s.n_tiles; ++kt) {
    lca::QWalk w;
    w.init(&s, kt, s.n_tiles);
    printf("K %d: %d %d\n", kt, w.t, w.t_end);
  }
  for (int t = 0; t < s.n_tiles; ++t)
    printf("T %d: %d %d\n", t, lca::token_tile(s, t, false), lca::token_tile(s, t, true));
  return 0;
}
