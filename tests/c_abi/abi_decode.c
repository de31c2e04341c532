/* A plain C client of libhq (include/hq.h), no Python or PyTorch: builds one
 * layer's hybrid cache in device memory, installs a 200-token prefix
 * (hq_select_vlines + hq_pack_merge in init mode), runs one decode step
 * (hq_decode_attn) and writes the inputs and the output to a file, so that a
 * test can replay the same inputs through the Python binding and compare.
 *
 *   usage: abi_decode <output file>
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "hq.h"

enum { B = 1, HQ = 8, HKV = 2, D = HQ_HEAD_DIM, W = 16, RHO_BP = 500, CAP = 256, VL_CAP = 16, L = 200, NQ = 64 };

/* float -> fp16 bits, round to nearest even (finite inputs of moderate size) */
static uint16_t to_half(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  int32_t e = (int32_t)((x >> 23) & 0xFF) - 127 + 15;
  uint32_t m = x & 0x7FFFFFu;
  if (e <= 0) {  /* subnormal half */
    if (e < -10) return (uint16_t)sign;
    m |= 0x800000u;
    const int shift = 14 - e;
    uint32_t h = m >> shift;
    const uint32_t rem = m & ((1u << shift) - 1u), half = 1u << (shift - 1);
    if (rem > half || (rem == half && (h & 1u))) ++h;
    return (uint16_t)(sign | h);
  }
  uint32_t h = ((uint32_t)e << 10) | (m >> 13);
  const uint32_t rem = m & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) ++h;
  return (uint16_t)(sign | h);
}

static uint64_t lcg = 0x2545F4914F6CDD1Dull;
static float uniform(void) {  /* [-2, 2) */
  lcg = lcg * 6364136223846793005ull + 1442695040888963407ull;
  return (float)((lcg >> 40) & 0xFFFFFF) / 16777216.0f * 4.0f - 2.0f;
}
static void fill(uint16_t* h, size_t n) {
  for (size_t i = 0; i < n; ++i) h[i] = to_half(uniform());
}

#define CK(x)                                                                \
  do {                                                                       \
    cudaError_t e_ = (x);                                                    \
    if (e_ != cudaSuccess) {                                                 \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));               \
      return 2;                                                              \
    }                                                                        \
  } while (0)
#define HQ(x)                                                                \
  do {                                                                       \
    hq_status s_ = (x);                                                      \
    if (s_ != HQ_OK) {                                                       \
      fprintf(stderr, "%s: %s (%s)\n", #x, hq_status_str(s_), hq_last_error()); \
      return 3;                                                              \
    }                                                                        \
  } while (0)

static void* dzero(size_t bytes) {
  void* p = NULL;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return NULL;
  cudaMemset(p, 0, bytes);
  return p;
}

int main(int argc, char** argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: abi_decode <output file>\n");
    return 1;
  }
  const int R = HQ_RING_LEN(W);
  hq_cache c;
  memset(&c, 0, sizeof c);
  c.B = B; c.Hq = HQ; c.Hkv = HKV; c.D = D; c.W = W; c.rho_bp = RHO_BP; c.cap = CAP; c.vl_cap = VL_CAP;
  c.pages = dzero((size_t)B * HKV * (CAP / 64) * HQ_PAGE_BYTES_KV(4, 4));
  c.kf = dzero((size_t)B * HKV * VL_CAP * D * 2);
  c.vf = dzero((size_t)B * HKV * VL_CAP * D * 2);
  c.vl_pos = dzero((size_t)B * HKV * VL_CAP * 4);
  c.kr = dzero((size_t)B * HKV * R * D * 2);
  c.vr = dzero((size_t)B * HKV * R * D * 2);
  c.qbuf = dzero((size_t)B * HQ * HQ_QBUF * D * 2);
  c.vl_sel = dzero((size_t)B * HKV * VL_CAP * 4);
  c.state = dzero((size_t)B * HQ_STATE_WORDS * 4);
  c.k_bits = 4;
  c.v_bits = 4;
  if (!c.pages || !c.kf || !c.vf || !c.vl_pos || !c.kr || !c.vr || !c.qbuf || !c.vl_sel || !c.state) return 2;
  HQ(hq_cache_validate(&c));

  /* inputs: prefix K, V [B, Hkv, L, D], the prompt's last NQ queries [B, Hq, NQ, D], one new token */
  const size_t nkv = (size_t)B * HKV * L * D, nqt = (size_t)B * HQ * NQ * D, nq1 = (size_t)B * HQ * D, nk1 = (size_t)B * HKV * D;
  uint16_t* host = malloc(2 * (2 * nkv + nqt + nq1 + 2 * nk1 + nq1));
  uint16_t *hk = host, *hv = hk + nkv, *hqt = hv + nkv, *hq1 = hqt + nqt, *hk1 = hq1 + nq1, *hv1 = hk1 + nk1, *hout = hv1 + nk1;
  fill(hk, nkv); fill(hv, nkv); fill(hqt, nqt); fill(hq1, nq1); fill(hk1, nk1); fill(hv1, nk1);
  uint16_t *dk = dzero(nkv * 2), *dv = dzero(nkv * 2), *dqt = dzero(nqt * 2), *dq1 = dzero(nq1 * 2), *dk1 = dzero(nk1 * 2),
           *dv1 = dzero(nk1 * 2), *dout = dzero(nq1 * 2);
  CK(cudaMemcpy(dk, hk, nkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dv, hv, nkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dqt, hqt, nqt * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dq1, hq1, nq1 * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dk1, hk1, nk1 * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dv1, hv1, nk1 * 2, cudaMemcpyHostToDevice));

  /* workspaces: zero-filled once, as hq.h asks */
  const size_t ws_sel = hq_workspace_bytes(&c, HQ_OP_SELECT, L), ws_mrg = hq_workspace_bytes(&c, HQ_OP_MERGE, L),
               ws_dec = hq_workspace_bytes(&c, HQ_OP_DECODE, 0);
  void *w_sel = dzero(ws_sel), *w_mrg = dzero(ws_mrg), *w_dec = dzero(ws_dec);

  HQ(hq_select_vlines(&c, dk, L, dqt, NQ, NULL, w_sel, ws_sel, NULL));
  HQ(hq_pack_merge(&c, dk, dv, L, w_mrg, ws_mrg, NULL));
  HQ(hq_decode_attn(&c, dq1, dk1, dv1, dout, 1.0f / sqrtf((float)D), w_dec, ws_dec, NULL));
  CK(cudaDeviceSynchronize());
  CK(cudaMemcpy(hout, dout, nq1 * 2, cudaMemcpyDeviceToHost));
  int32_t st[HQ_STATE_WORDS];
  CK(cudaMemcpy(st, c.state, sizeof st, cudaMemcpyDeviceToHost));
  if (st[HQ_STATE_T] != L + 1 || st[HQ_STATE_ERR] != 0) {
    fprintf(stderr, "state after the step: T=%d err=%d\n", st[HQ_STATE_T], st[HQ_STATE_ERR]);
    return 4;
  }
  FILE* f = fopen(argv[1], "wb");
  if (!f) return 5;
  fwrite(host, 2, 2 * nkv + nqt + nq1 + 2 * nk1 + nq1, f);
  fclose(f);
  printf("abi_decode ok: T=%d n_packed=%d n_vl=%d\n", st[HQ_STATE_T], st[HQ_STATE_NPACKED], st[HQ_STATE_NVL]);
  return 0;
}
