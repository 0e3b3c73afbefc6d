/*
 * A plain C caller of libep: the hand-worked 2-rank, 3-token routing example
 * (tests/golden/routing_tiny.json) through ep_get_dispatch_layout,
 * ep_dispatch and ep_combine, then through the low-latency pair
 * ep_ll_dispatch (bf16 payload) and ep_ll_combine with identity experts, with
 * device buffers from cudaMalloc and the default stream.  The example's rows have 2 channels; the library moves rows
 * of a multiple of 8 channels (16 bytes), so each row is zero-padded to 8
 * channels and only the example's 2 are printed.  Prints every output as
 * "name v0 v1 ..." lines for the test to compare with the fixture.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#include "ep.h"

#define R 2
#define T 3
#define K 2
#define E 4
#define HX 2 /* the example's channels */
#define H 8  /* channels per row as stored (zero-padded) */
#define CAP (R * T)
#define EL (E / R)

#define CK(x)                                                                  \
  do {                                                                         \
    if ((x) != cudaSuccess) {                                                  \
      fprintf(stderr, "cuda error at %s:%d\n", __FILE__, __LINE__);           \
      return 1;                                                                \
    }                                                                          \
  } while (0)
#define EK(x)                                                                  \
  do {                                                                         \
    int rc_ = (x);                                                             \
    if (rc_ != EP_OK) {                                                        \
      fprintf(stderr, "ep error %d (%s) at %s:%d\n", rc_, ep_status_string(rc_), \
              __FILE__, __LINE__);                                             \
      return 1;                                                                \
    }                                                                          \
  } while (0)

static unsigned short bf16(float f) {
  unsigned int u;
  memcpy(&u, &f, 4);
  return (unsigned short)(u >> 16); /* the example's values are exact in bf16 */
}

static void print_i32(const char *name, const int *v, int n) {
  printf("%s", name);
  for (int i = 0; i < n; ++i) printf(" %d", v[i]);
  printf("\n");
}

int main(void) {
  const int64_t idx_h[R * T * K] = {1, 2, 0, -1, 3, 2, -1, -1, 2, 0, 1, 1};
  const float w_h[R * T * K] = {0.25f, 0.75f, 1.0f, 0.5f, 0.625f, 0.375f,
                                0.5f,  0.5f,  0.125f, 0.875f, 0.3125f, 0.6875f};
  const float xf[R * T * HX] = {1.0f, -2.0f, 0.5f, 3.0f, 1.5f, 0.25f,
                               7.0f, 7.0f,  -1.0f, 2.5f, 0.125f, -0.5f};
  unsigned short x_h[R * T * H];
  memset(x_h, 0, sizeof x_h);
  for (int t = 0; t < R * T; ++t)
    for (int c = 0; c < HX; ++c) x_h[t * H + c] = bf16(xf[t * HX + c]);

  int64_t *idx;
  float *w, *rw, *cw;
  void *x, *rx, *cx, *ws;
  int *ntpr, *ntpe, *P, *rc, *nrte, *sp, *rsi, *st;
  int64_t *ri;
  unsigned char *inr;
  const size_t wsb = ep_dispatch_workspace_bytes(R, T, E);
  CK(cudaMalloc((void **)&idx, sizeof idx_h));
  CK(cudaMalloc((void **)&w, sizeof w_h));
  CK(cudaMalloc(&x, sizeof x_h));
  CK(cudaMalloc((void **)&ntpr, R * R * 4));
  CK(cudaMalloc((void **)&ntpe, R * E * 4));
  CK(cudaMalloc((void **)&inr, R * T * R));
  CK(cudaMalloc(&rx, R * CAP * H * 2));
  CK(cudaMalloc((void **)&ri, R * CAP * K * 8));
  CK(cudaMalloc((void **)&rw, R * CAP * K * 4));
  CK(cudaMalloc((void **)&rsi, R * CAP * 4));
  CK(cudaMalloc((void **)&P, R * R * 4));
  CK(cudaMalloc((void **)&rc, R * 4));
  CK(cudaMalloc((void **)&nrte, E * 4));
  CK(cudaMalloc((void **)&sp, R * T * R * 4));
  CK(cudaMalloc(&cx, R * T * H * 2));
  CK(cudaMalloc((void **)&cw, R * T * K * 4));
  CK(cudaMalloc(&ws, wsb));
  CK(cudaMalloc((void **)&st, 4));
  CK(cudaMemset(st, 0, 4));
  CK(cudaMemcpy(idx, idx_h, sizeof idx_h, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(w, w_h, sizeof w_h, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(x, x_h, sizeof x_h, cudaMemcpyHostToDevice));

  EK(ep_get_dispatch_layout(idx, R, T, K, E, R, ntpr, ntpe, inr, st, 0));
  EK(ep_dispatch(x, idx, w, inr, R, T, H, K, E, 1, CAP, rx, ri, rw, rsi, P, rc, nrte, sp, ws,
                 wsb, st, 0));
  EK(ep_combine(rx, rw, sp, NULL, NULL, R, T, H, K, CAP, cx, cw, st, 0));
  CK(cudaDeviceSynchronize());

  int ntpr_h[R * R], ntpe_h[R * E], P_h[R * R], rc_h[R], nrte_h[E], sp_h[R * T * R],
      rsi_h[R * CAP], st_h;
  unsigned char inr_h[R * T * R];
  int64_t ri_h[R * CAP * K];
  float rw_h[R * CAP * K], cw_h[R * T * K];
  unsigned short cx_h[R * T * H];
  CK(cudaMemcpy(ntpr_h, ntpr, sizeof ntpr_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(ntpe_h, ntpe, sizeof ntpe_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(inr_h, inr, sizeof inr_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(P_h, P, sizeof P_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(rc_h, rc, sizeof rc_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(nrte_h, nrte, sizeof nrte_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(sp_h, sp, sizeof sp_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(rsi_h, rsi, sizeof rsi_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(ri_h, ri, sizeof ri_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(rw_h, rw, sizeof rw_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(cx_h, cx, sizeof cx_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(cw_h, cw, sizeof cw_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&st_h, st, 4, cudaMemcpyDeviceToHost));

  int inr_i[R * T * R];
  for (int i = 0; i < R * T * R; ++i) inr_i[i] = inr_h[i];
  print_i32("status", &st_h, 1);
  print_i32("num_tokens_per_rank", ntpr_h, R * R);
  print_i32("num_tokens_per_expert", ntpe_h, R * E);
  print_i32("is_token_in_rank", inr_i, R * T * R);
  print_i32("rank_prefix_matrix", P_h, R * R);
  print_i32("recv_count", rc_h, R);
  print_i32("num_recv_tokens_per_expert", nrte_h, E);
  print_i32("send_pos", sp_h, R * T * R);
  for (int d = 0; d < R; ++d) {
    printf("recv_src_idx_%d", d);
    for (int r = 0; r < rc_h[d]; ++r) printf(" %d", rsi_h[d * CAP + r]);
    printf("\nrecv_topk_idx_%d", d);
    for (int r = 0; r < rc_h[d]; ++r)
      for (int k = 0; k < K; ++k) printf(" %lld", (long long)ri_h[(d * CAP + r) * K + k]);
    printf("\nrecv_topk_weights_%d", d);
    for (int r = 0; r < rc_h[d]; ++r)
      for (int k = 0; k < K; ++k) printf(" %.9g", rw_h[(d * CAP + r) * K + k]);
    printf("\n");
  }
  printf("combined_x");
  for (int t = 0; t < R * T; ++t)
    for (int c = 0; c < HX; ++c) {
      unsigned int u = (unsigned int)cx_h[t * H + c] << 16;
      float f;
      memcpy(&f, &u, 4);
      printf(" %.9g", f);
    }
  printf("\ncombined_topk_weights");
  for (int i = 0; i < R * T * K; ++i) printf(" %.9g", cw_h[i]);
  printf("\n");

  /* low latency: bf16 slabs [R, E_l, R*T, H], then the weighted combine of
     the slab rows as they are (identity experts) */
  void *slab, *lout, *lws;
  int *lrc, *lrsi, *llr, *lpos;
  const size_t lwsb = ep_ll_workspace_bytes(R, T, E);
  CK(cudaMalloc(&slab, (size_t)R * EL * CAP * H * 2));
  CK(cudaMalloc(&lout, R * T * H * 2));
  CK(cudaMalloc(&lws, lwsb));
  CK(cudaMalloc((void **)&lrc, R * EL * 4));
  CK(cudaMalloc((void **)&lrsi, R * EL * CAP * 4));
  CK(cudaMalloc((void **)&llr, R * EL * R * 2 * 4));
  CK(cudaMalloc((void **)&lpos, R * T * K * 4));
  EK(ep_ll_dispatch(x, idx, NULL, R, T, H, K, E, 0, slab, NULL, lrc, lrsi, llr, lpos, NULL, lws,
                    lwsb, st, 0));
  EK(ep_ll_combine(slab, idx, w, lpos, NULL, R, T, H, K, E, lout, st, 0));
  CK(cudaDeviceSynchronize());
  int lrc_h[R * EL], lrsi_h[R * EL * CAP], llr_h[R * EL * R * 2], lpos_h[R * T * K];
  unsigned short slab_h[R * EL * CAP * H], lout_h[R * T * H];
  CK(cudaMemcpy(lrc_h, lrc, sizeof lrc_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(lrsi_h, lrsi, sizeof lrsi_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(llr_h, llr, sizeof llr_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(lpos_h, lpos, sizeof lpos_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(slab_h, slab, sizeof slab_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(lout_h, lout, sizeof lout_h, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&st_h, st, 4, cudaMemcpyDeviceToHost));
  print_i32("ll_status", &st_h, 1);
  print_i32("ll_recv_count", lrc_h, R * EL);
  print_i32("ll_layout_range", llr_h, R * EL * R * 2);
  print_i32("ll_pos", lpos_h, R * T * K);
  for (int e = 0; e < R * EL; ++e) {
    printf("ll_recv_src_info_%d_%d", e / EL, e % EL);
    for (int r = 0; r < lrc_h[e]; ++r) printf(" %d", lrsi_h[e * CAP + r]);
    printf("\nll_slab_%d_%d", e / EL, e % EL);
    for (int r = 0; r < lrc_h[e]; ++r)
      for (int c = 0; c < HX; ++c) {
        unsigned int u = (unsigned int)slab_h[(e * CAP + r) * H + c] << 16;
        float f;
        memcpy(&f, &u, 4);
        printf(" %.9g", f);
      }
    printf("\n");
  }
  printf("ll_combined_x");
  for (int t = 0; t < R * T; ++t)
    for (int c = 0; c < HX; ++c) {
      unsigned int u = (unsigned int)lout_h[t * H + c] << 16;
      float f;
      memcpy(&f, &u, 4);
      printf(" %.9g", f);
    }
  printf("\n");
  return 0;
}
