// Host-side probe of index logic the kernels share with the host: the
// feedforward tile raster (ffn_sm100.cuh) and the packed-sequence view
// (sched.cuh).  Built and run by tests/test_layout_host.py.
//   layout_probe tiles n_tm n_tn group_m -> "t tm tn" per tile
//   layout_probe seq S_max tile S_tensor cu0 cu1 ...  -> "b ok tokb len n_tiles"
//   layout_probe s2 S half H first_shifted -> "h p token" per head and position
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include <cuda.h>

#include "../../long_context_exact_attention_b200/csrc/aux_kernels.cuh"
#include "../../long_context_exact_attention_b200/csrc/ffn_sm100.cuh"
#include "../../long_context_exact_attention_b200/csrc/sched.cuh"

int main(int argc, char** argv) {
  if (argc < 2) return 2;
  if (!strcmp(argv[1], "tiles")) {
    const int n_tm = atoi(argv[2]), n_tn = atoi(argv[3]), group_m = atoi(argv[4]);
    for (int t = 0; t < n_tm * n_tn; ++t) {
      int tm, tn;
      lca::ffn::tile_coords(t, n_tm, n_tn, group_m, tm, tn);
      printf("%d %d %d\n", t, tm, tn);
    }
    return 0;
  }
  if (!strcmp(argv[1], "seq")) {
    lca::AttnSched s;
    memset(&s, 0, sizeof s);
    s.S = atoi(argv[2]);
    s.tile = atoi(argv[3]);
    s.n_tiles = (s.S + s.tile - 1) / s.tile;
    const int S_tensor = atoi(argv[4]);
    std::vector<int> cu;
    for (int i = 5; i < argc; ++i) cu.push_back(atoi(argv[i]));
    s.cu_seqlens = cu.data();
    for (int b = 0; b + 1 < static_cast<int>(cu.size()); ++b) {
      lca::SeqView v{};
      const bool ok = lca::seq_view(s, b, S_tensor, &v);
      printf("%d %d %d %d %d\n", b, ok ? 1 : 0, v.tokb, v.len, v.n_tiles);
    }
    return 0;
  }
  if (!strcmp(argv[1], "s2")) {
    const int S = atoi(argv[2]), half = atoi(argv[3]), H = atoi(argv[4]), first = atoi(argv[5]);
    for (int h = 0; h < H; ++h)
      for (int p = 0; p < S; ++p) printf("%d %d %d\n", h, p, lca::s2_token(p, h, first, half, S));
    return 0;
  }
  return 2;
}
