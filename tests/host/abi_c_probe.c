/* Plain C client of liblca (include/lca.h), built with gcc by
 * tests/test_abi_c.py: the library is usable from C with nothing but the
 * header, the shared library and the CUDA runtime.
 *
 *   abi_c_probe cpu   -- status strings, version, synchronous argument
 *                        errors (no GPU needed)
 *   abi_c_probe gpu   -- a causal bf16 forward whose answer is a closed
 *                        form: with all-zero keys every logit is 0, so row
 *                        i of the output is the mean of v_0..v_i and
 *                        lse_i = ln(i + 1)
 * Exit status 0 on success; prints what failed otherwise. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "lca.h"

static int fails = 0;
#define CHECK(cond, ...)                \
  do {                                  \
    if (!(cond)) {                      \
      fprintf(stderr, __VA_ARGS__);     \
      fprintf(stderr, "\n");            \
      ++fails;                          \
    }                                   \
  } while (0)

static uint16_t to_bf16(float x) { /* round to nearest even; inputs are finite */
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static float from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

static int cpu_checks(void) {
  CHECK(strcmp(lca_status_string(LCA_OK), "LCA_OK") == 0, "status string of LCA_OK");
  CHECK(strcmp(lca_status_string(LCA_ERR_WORKSPACE), "LCA_ERR_WORKSPACE") == 0,
        "status string of LCA_ERR_WORKSPACE");
  CHECK((lca_version() >> 16) == 1, "major version");
  lca_shape sh = {1, 4, 2, 256, 128, LCA_BF16, 0.0f};
  void* fake = (void*)(uintptr_t)0x10000; /* aligned, never dereferenced */
  /* bad shapes and pointers come back synchronously, before any launch */
  lca_shape bad = sh;
  bad.Hq = 3;
  CHECK(lca_attn_fwd(&bad, fake, fake, fake, 1, 0, NULL, fake, (float*)fake, NULL) ==
            LCA_ERR_INVALID_ARG, "Hq %% Hkv != 0 accepted");
  bad = sh;
  bad.d = 64;
  CHECK(lca_attn_fwd(&bad, fake, fake, fake, 1, 0, NULL, fake, (float*)fake, NULL) ==
            LCA_ERR_UNSUPPORTED, "bf16 d = 64 accepted");
  CHECK(lca_attn_fwd(&sh, NULL, fake, fake, 1, 0, NULL, fake, (float*)fake, NULL) ==
            LCA_ERR_INVALID_ARG, "NULL q accepted");
  CHECK(strlen(lca_last_error()) > 0, "no error detail");
  CHECK(lca_attn_bwd_workspace_size(&sh) > 0, "workspace size of a valid shape");
  lca_ffn_shape fs = {300, 256, 384};
  CHECK(lca_ffn_workspace_size(&fs, 128) == (size_t)128 * 384 * 2, "feedforward workspace");
  return fails;
}

static int gpu_checks(void) {
  const int S = 300, H = 2, D = 128; /* ragged: 300 is not a multiple of 128 */
  const size_t n = (size_t)S * H * D;
  uint16_t* hq = malloc(n * 2);
  uint16_t* hk = malloc(n * 2);
  uint16_t* hv = malloc(n * 2);
  uint16_t* ho = malloc(n * 2);
  float* hl = malloc((size_t)H * S * 4);
  for (size_t i = 0; i < n; ++i) {
    hq[i] = to_bf16((float)((int)(i % 13) - 6) * 0.25f);
    hk[i] = 0; /* zero keys: every logit is 0 */
    hv[i] = to_bf16((float)((int)((i * 7) % 17) - 8) * 0.125f);
  }
  void *dq, *dk, *dv, *dout;
  float* dl;
  if (cudaMalloc(&dq, n * 2) || cudaMalloc(&dk, n * 2) || cudaMalloc(&dv, n * 2) ||
      cudaMalloc(&dout, n * 2) || cudaMalloc((void**)&dl, (size_t)H * S * 4)) {
    fprintf(stderr, "cudaMalloc failed\n");
    return 1;
  }
  cudaMemcpy(dq, hq, n * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dk, hk, n * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dv, hv, n * 2, cudaMemcpyHostToDevice);
  lca_shape sh = {1, H, H, S, D, LCA_BF16, 0.0f};
  lca_opts o = {LCA_ORDER_RING, NULL, 0, 0};
  CHECK(lca_attn_fwd(&sh, dq, dk, dv, 1, 128, &o, dout, dl, NULL) == LCA_OK, "forward: %s",
        lca_last_error());
  CHECK(lca_check(NULL) == LCA_OK, "lca_check: %s", lca_last_error());
  cudaMemcpy(ho, dout, n * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(hl, dl, (size_t)H * S * 4, cudaMemcpyDeviceToHost);
  double max_o = 0.0, max_l = 0.0;
  for (int h = 0; h < H; ++h) {
    for (int c = 0; c < D; ++c) {
      double run = 0.0;
      for (int i = 0; i < S; ++i) {
        run += from_bf16(hv[((size_t)i * H + h) * D + c]);
        const double want = run / (i + 1);
        const double got = from_bf16(ho[((size_t)i * H + h) * D + c]);
        if (fabs(got - want) > max_o) max_o = fabs(got - want);
      }
    }
    for (int i = 0; i < S; ++i) {
      const double e = fabs(hl[(size_t)h * S + i] - log((double)(i + 1)));
      if (e > max_l) max_l = e;
    }
  }
  /* P = 1/(i+1) is rounded to bf16 before P V; lse is fp32 */
  CHECK(max_o <= 2e-2, "output off the running mean by %g", max_o);
  CHECK(max_l <= 1e-3, "lse off ln(i+1) by %g", max_l);
  printf("max |out - mean| %g, max |lse - ln(i+1)| %g\n", max_o, max_l);

  /* The same attention as two ring steps through the block entry points:
   * keys [0, 128) then keys [128, 300) (a ragged block whose diagonal
   * starts one tile in), folded into a running float32 (O, lse). */
  float *oacc, *lacc;
  void* dout2;
  if (cudaMalloc((void**)&oacc, n * 4) || cudaMalloc((void**)&lacc, (size_t)H * S * 4) ||
      cudaMalloc(&dout2, n * 2)) {
    fprintf(stderr, "cudaMalloc failed\n");
    return 1;
  }
  const size_t row = (size_t)H * D; /* elements per token */
  lca_block_shape b1 = {1, H, H, S, 128, D, LCA_BF16, 0.0f};
  lca_block_shape b2 = {1, H, H, S, S - 128, D, LCA_BF16, 0.0f};
  CHECK(lca_attn_fwd_block(&b1, dq, dk, dv, 1, 0, 0, 0, oacc, lacc, NULL, NULL) == LCA_OK,
        "first block: %s", lca_last_error());
  CHECK(lca_attn_fwd_block(&b2, dq, (uint16_t*)dk + 128 * row, (uint16_t*)dv + 128 * row, 1, 0,
                           128, 1, oacc, lacc, dout2, NULL) == LCA_OK,
        "second block: %s", lca_last_error());
  CHECK(lca_check(NULL) == LCA_OK, "lca_check: %s", lca_last_error());
  cudaMemcpy(ho, dout2, n * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(hl, lacc, (size_t)H * S * 4, cudaMemcpyDeviceToHost);
  max_o = 0.0;
  max_l = 0.0;
  for (int h = 0; h < H; ++h) {
    for (int c = 0; c < D; ++c) {
      double run = 0.0;
      for (int i = 0; i < S; ++i) {
        run += from_bf16(hv[((size_t)i * H + h) * D + c]);
        const double got = from_bf16(ho[((size_t)i * H + h) * D + c]);
        if (fabs(got - run / (i + 1)) > max_o) max_o = fabs(got - run / (i + 1));
      }
    }
    for (int i = 0; i < S; ++i) {
      const double e = fabs(hl[(size_t)h * S + i] - log((double)(i + 1)));
      if (e > max_l) max_l = e;
    }
  }
  CHECK(max_o <= 2e-2, "block output off the running mean by %g", max_o);
  CHECK(max_l <= 1e-3, "block lse off ln(i+1) by %g", max_l);
  printf("blocks: max |out - mean| %g, max |lse - ln(i+1)| %g\n", max_o, max_l);
  cudaFree(oacc);
  cudaFree(lacc);
  cudaFree(dout2);
  cudaFree(dq);
  cudaFree(dk);
  cudaFree(dv);
  cudaFree(dout);
  cudaFree(dl);
  free(hq);
  free(hk);
  free(hv);
  free(ho);
  free(hl);
  return fails;
}

int main(int argc, char** argv) {
  if (argc < 2) return 2;
  const int r = strcmp(argv[1], "gpu") == 0 ? gpu_checks() : cpu_checks();
  if (r == 0) printf("ok\n");
  return r ? 1 : 0;
}
