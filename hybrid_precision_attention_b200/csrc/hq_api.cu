// hq_api.cu — the extern "C" entry points of libhq.so (declared in include/hq.h).
//
// Host-side argument validation happens here, before anything is launched;
// the kernels live in decode.cu, select.cu, pack_merge.cu and prefill.cu.
#include <cuda_runtime.h>

#include <cstdio>

#include "common.cuh"

namespace hq {
hq_status launch_clear_bitmaps(const hq_cache& c, int sms, cudaStream_t st);
hq_status launch_pack_merge(const hq_cache& c, const uint16_t* kd, const uint16_t* vd, int L, void* ws, cudaStream_t st);
hq_status launch_decode(const hq_cache& c, const uint16_t* q, const uint16_t* kn, const uint16_t* vn, uint16_t* out,
                        float sm_scale, void* ws, int sms, cudaStream_t st);
size_t decode_workspace(const hq_cache& c, int sms);
bool decode_supported(const hq_cache& c);
size_t select_workspace(const hq_cache& c, bool need_scores);
hq_status launch_select(const hq_cache& c, const uint16_t* kd, int L, const uint16_t* qe, int nq, float* scores_out,
                        void* ws, cudaStream_t st);
size_t prefill_workspace(int B, int Hq, int Hkv, int L, int vl_stride);
hq_status launch_prefill(int B, int Hq, int Hkv, int L, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* vl_pos, int n_vl, int vl_stride, int W, int qk_format, float sm_scale,
                         uint16_t* out, void* ws, cudaStream_t st);
}  // namespace hq

namespace {

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return sms;
}

}  // namespace

namespace hq {
thread_local char g_last_error[256] = "";
hq_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return HQ_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorName(e));
  return HQ_ERR_CUDA;
}
hq_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, e == cudaSuccess ? "driver call failed" : cudaGetErrorName(e));
  return HQ_ERR_CUDA;
}
}  // namespace hq

extern "C" {

const char* hq_last_error(void) { return hq::g_last_error; }


int32_t hq_abi_version(void) { return HQ_ABI_VERSION; }

const char* hq_status_str(hq_status s) {
  switch (s) {
    case HQ_OK: return "ok";
    case HQ_ERR_INVALID: return "invalid argument";
    case HQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case HQ_ERR_WORKSPACE: return "workspace missing or too small";
    case HQ_ERR_CAPACITY: return "capacity exceeded";
    case HQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

hq_status hq_cache_validate(const hq_cache* c) {
  if (!c) return HQ_ERR_INVALID;
  if (c->D != HQ_HEAD_DIM) return HQ_ERR_UNSUPPORTED;
  if (c->B <= 0 || c->Hq <= 0 || c->Hkv <= 0 || c->Hq % c->Hkv != 0) return HQ_ERR_INVALID;
  if (c->Hq / c->Hkv > HQ_MAX_GQA) return HQ_ERR_UNSUPPORTED;
  if (c->W < 0 || c->rho_bp < 0 || c->rho_bp > 10000) return HQ_ERR_INVALID;
  if (c->cap <= 0 || c->cap % 128 != 0 || c->vl_cap <= 0 || c->vl_cap % 16 != 0) return HQ_ERR_INVALID;
  if (c->B > 65535 || c->Hkv > 65535) return HQ_ERR_UNSUPPORTED;
  const void* ptrs[] = {c->pages, c->kf, c->vf, c->vl_pos, c->kr, c->vr, c->qbuf, c->vl_sel, c->state};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HQ_ERR_INVALID;
  if (c->page_table != nullptr && ((reinterpret_cast<uintptr_t>(c->page_table) & 3u) != 0 || c->n_pages < 1))
    return HQ_ERR_INVALID;
  if (c->score_acc != nullptr && (reinterpret_cast<uintptr_t>(c->score_acc) & 15u) != 0) return HQ_ERR_INVALID;
  if (c->qlse != nullptr && (reinterpret_cast<uintptr_t>(c->qlse) & 15u) != 0) return HQ_ERR_INVALID;
  {
    const int kb = c->k_bits ? c->k_bits : 4, vb = c->v_bits ? c->v_bits : 4;
    if ((kb != 2 && kb != 4 && kb != 8) || (vb != 2 && vb != 4 && vb != 8)) return HQ_ERR_INVALID;
    if (!((kb == 4 && vb == 4) || (kb == 8 && vb == 8) || (kb == 4 && vb == 2) || (kb == 2 && vb == 4)))
      return HQ_ERR_UNSUPPORTED;
  }
  return HQ_OK;
}

size_t hq_workspace_bytes(const hq_cache* c, int32_t op, int32_t L) {
  if (hq_cache_validate(c) != HQ_OK) return 0;
  switch (op) {
    case HQ_OP_SELECT: {
      hq_cache t = *c;
      if (L > t.cap) t.cap = ((L + 127) / 128) * 128;
      return hq::select_workspace(t, true);
    }
    case HQ_OP_MERGE: return 256 + 2ull * c->B * c->Hkv * c->vl_cap * HQ_HEAD_DIM * 2;
    case HQ_OP_DECODE: return hq::decode_workspace(*c, sm_count());
  }
  return 0;
}

hq_status hq_cache_reset(const hq_cache* c, hq_stream_t stream) {
  hq_status s = hq_cache_validate(c);
  if (s != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(c->state, 0, static_cast<size_t>(c->B) * HQ_STATE_WORDS * sizeof(int32_t), st);
  if (e != cudaSuccess) return hq::cuda_status(e, "reset state");
  if (c->score_acc != nullptr) {
    e = cudaMemsetAsync(c->score_acc, 0, static_cast<size_t>(c->B) * c->Hkv * c->cap * sizeof(float), st);
    if (e != cudaSuccess) return hq::cuda_status(e, "reset running scores");
  }
  return hq::launch_clear_bitmaps(*c, sm_count(), st);
}

hq_status hq_select_vlines(const hq_cache* c, const uint16_t* k_dense, int32_t L, const uint16_t* q_ext, int32_t nq,
                           float* scores_out, void* ws, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = hq_cache_validate(c);
  if (s != HQ_OK) return s;
  const bool init = k_dense != nullptr;
  if (init) {
    if (!aligned16(k_dense) || !aligned16(q_ext)) return HQ_ERR_INVALID;
    if (L <= 0 || nq < 1 || nq > HQ_QBUF || nq > L) return HQ_ERR_INVALID;
    if (L > c->cap) return HQ_ERR_CAPACITY;
  } else if (q_ext != nullptr) {
    return HQ_ERR_INVALID;
  }
  if (scores_out && !aligned16(scores_out)) return HQ_ERR_INVALID;
  if (!aligned16(ws) || ws_bytes < hq::select_workspace(*c, true)) return HQ_ERR_WORKSPACE;
  return hq::launch_select(*c, k_dense, init ? L : 0, q_ext, init ? nq : 0, scores_out, ws,
                           reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_pack_merge(const hq_cache* c, const uint16_t* k_dense, const uint16_t* v_dense, int32_t L, void* ws,
                        size_t ws_bytes, hq_stream_t stream) {
  hq_status s = hq_cache_validate(c);
  if (s != HQ_OK) return s;
  const bool init = k_dense != nullptr || v_dense != nullptr;
  if (init) {
    if (!aligned16(k_dense) || !aligned16(v_dense)) return HQ_ERR_INVALID;
    if (L <= 0) return HQ_ERR_INVALID;
    if (L > c->cap) return HQ_ERR_CAPACITY;
  }
  if (!aligned16(ws) || ws_bytes < hq_workspace_bytes(c, HQ_OP_MERGE, 0)) return HQ_ERR_WORKSPACE;
  return hq::launch_pack_merge(*c, k_dense, v_dense, init ? L : 0, ws, reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_decode_attn(const hq_cache* c, const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                         uint16_t* out, float sm_scale, void* ws, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = hq_cache_validate(c);
  if (s != HQ_OK) return s;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return HQ_ERR_INVALID;
  if (!(sm_scale > 0.0f)) return HQ_ERR_INVALID;
  if (!hq::decode_supported(*c)) return HQ_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (!aligned16(ws) || ws_bytes < hq::decode_workspace(*c, sms)) return HQ_ERR_WORKSPACE;
  return hq::launch_decode(*c, q, k_new, v_new, out, sm_scale, ws, sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t L, int32_t D, int32_t vl_stride) {
  if (D != HQ_HEAD_DIM || B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || Hq % Hkv || vl_stride < 0) return 0;
  return hq::prefill_workspace(B, Hq, Hkv, L, vl_stride);
}

hq_status hq_prefill_attn(int32_t B, int32_t Hq, int32_t Hkv, int32_t L, int32_t D, const uint16_t* q,
                          const uint16_t* k, const uint16_t* v, const int32_t* vl_pos, int32_t n_vl, int32_t vl_stride,
                          int32_t W, int32_t qk_format, float sm_scale, uint16_t* out, void* ws, size_t ws_bytes,
                          hq_stream_t stream) {
  if (qk_format != HQ_PREFILL_E4M3 && qk_format != HQ_PREFILL_INT8_QK) return HQ_ERR_INVALID;
  if (D != HQ_HEAD_DIM) return HQ_ERR_UNSUPPORTED;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L <= 0 || W < 0 || !(sm_scale > 0.0f)) return HQ_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return HQ_ERR_INVALID;
  if (n_vl < 0 || n_vl > vl_stride || (n_vl > 0 && !aligned16(vl_pos))) return HQ_ERR_INVALID;
  if (!aligned16(ws) || ws_bytes < hq::prefill_workspace(B, Hq, Hkv, L, vl_stride)) return HQ_ERR_WORKSPACE;
  return hq::launch_prefill(B, Hq, Hkv, L, q, k, v, vl_pos, n_vl, vl_stride, W, qk_format, sm_scale, out, ws,
                            reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
