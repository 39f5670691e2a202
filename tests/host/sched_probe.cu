// Host-side probe of the tile walks in sched.cuh: prints, for the schedule
// given on the command line, every query tile's key/value tile sequence and
// every key tile's query tile range.  Built and run by tests/test_sched_host.py.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../long_context_exact_attention_b200/csrc/sched.cuh"

int main(int argc, char** argv) {
  // args: n_tiles causal s2 tiles_per_chunk n_chunks order q_block_tiles group_tiles
  //       shift_tiles first_shifted_head [perm...]
  if (argc < 11) return 2;
  lca::AttnSched s;
  std::memset(&s, 0, sizeof s);
  s.n_tiles = atoi(argv[1]);
  s.causal = atoi(argv[2]);
  s.s2 = atoi(argv[3]);
  s.tiles_per_chunk = atoi(argv[4]);
  s.n_chunks = atoi(argv[5]);
  s.order = atoi(argv[6]);
  s.q_block_tiles = atoi(argv[7]);
  s.group_tiles = atoi(argv[8]);
  s.shift_tiles = atoi(argv[9]);
  s.first_shifted_head = atoi(argv[10]);
  for (int i = 11; i < argc && i - 11 < LCA_MAX_CHUNKS; ++i) s.perm[i - 11] = atoi(argv[i]);
  for (int qt = 0; qt < s.n_tiles; ++qt) {
    lca::KvWalk w;
    w.init(&s, qt);
    printf("Q %d:", qt);
    int t;
    while (w.next(t)) printf(" %d", t);
    printf("\n");
  }
  for (int kt = 0; kt < s.n_tiles; ++kt) {
    lca::QWalk w;
    w.init(&s, kt);
    printf("K %d: %d %d\n", kt, w.t, w.t_end);
  }
  for (int t = 0; t < s.n_tiles; ++t)
    printf("T %d: %d %d\n", t, lca::token_tile(s, t, false), lca::token_tile(s, t, true));
  return 0;
}
