// decode_noalloc.cu — hq_decode_attn_noalloc: the decode step for callers that
// must not allocate device memory.
//
// hq_decode_attn needs a caller-provided workspace (split-K partials and
// completion counters).  Some callers cannot obtain one: a plugin running inside
// a serving engine that owns every byte of device memory and forbids allocation
// once it is up, or a latency-critical loop where cudaMalloc / cudaFree would
// synchronise the device.  This entry point takes its workspace from a fixed
// scratch array compiled into the library instead.
//
//   * The scratch is a file-scope __device__ array of HQ_NOALLOC_SCRATCH_BYTES
//     (4 MiB).  Every GPU on which the library is loaded holds one copy until the
//     process exits.
//   * Host code cannot use the array's name as a device address, so the first
//     call on each device (with that device current) looks the address up with
//     cudaGetSymbolAddress and remembers it, together with the id of the
//     device's current context.  A later call that finds a different context
//     (the device was reset, or its primary context released and created
//     again, which reloads the library's device code) looks it up again.  Make
//     the first call on a device, and the first call after such a reset,
//     before any stream capture.
//   * All calls on a device share the one array and it keeps whatever the last
//     call left in it: each call clears the completion counters (an async
//     memset on the caller's stream) before the kernel.  Two calls whose
//     executions overlap on the GPU (different streams, no ordering) race on
//     the array and must not be issued.
//   * No allocation happens here: no cudaMalloc, cudaFree or allocating library
//     routine.  A cache whose decode workspace would exceed the array is
//     rejected with HQ_ERR_WORKSPACE before anything is launched.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace hq {
hq_status launch_decode(const hq_cache& c, const uint16_t* q, const uint16_t* kn, const uint16_t* vn, uint16_t* out,
                        float sm_scale, void* ws, int sms, cudaStream_t st);
size_t decode_workspace(const hq_cache& c, int sms);
size_t decode_counter_bytes(const hq_cache& c);
bool decode_supported(const hq_cache& c);
}  // namespace hq

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context (0 when it cannot be read, in
// which case the address found first is kept).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr && get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of this device's scratch array (looked up once per device
// and context).
hq_status scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr || (ctx != 0 && ctx != g_scratch_ctx[dev])) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return hq::cuda_fail(e, "scratch address");
    g_scratch_addr[dev] = p;
    // the lookup made the device's context current if no call had yet: record its id
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *out = g_scratch_addr[dev];
  return HQ_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" HQ_API hq_status hq_decode_attn_noalloc(const hq_cache* c, const uint16_t* q, const uint16_t* k_new,
                                                   const uint16_t* v_new, uint16_t* out, float sm_scale,
                                                   hq_stream_t stream) {
  hq_status s = hq_cache_validate(c);
  if (s != HQ_OK) return s;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return HQ_ERR_INVALID;
  if (!(sm_scale > 0.0f)) return HQ_ERR_INVALID;
  if (!hq::decode_supported(*c)) return HQ_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return hq::cuda_fail(e, "device query");
  if (hq::decode_workspace(*c, sms) > HQ_NOALLOC_SCRATCH_BYTES) return HQ_ERR_WORKSPACE;
  void* ws = nullptr;
  s = scratch_address(dev, &ws);
  if (s != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the counters must start at zero; the rest of the scratch is written before it is read
  e = cudaMemsetAsync(ws, 0, hq::decode_counter_bytes(*c), st);
  if (e != cudaSuccess) return hq::cuda_fail(e, "counter reset");
  return hq::launch_decode(*c, q, k_new, v_new, out, sm_scale, ws, sms, st);
}
