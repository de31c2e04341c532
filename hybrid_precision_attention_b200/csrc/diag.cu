// diag.cu — measurement helper with no counterpart in the method: a read-only
// HBM streaming kernel, used to measure the bandwidth ceiling that a kernel
// which only reads (like the decode scan) can reach on this GPU.  A copy
// benchmark moves every byte twice (read + write) and so measures a different
// mix of DRAM traffic.
#include <cuda_runtime.h>

#include "common.cuh"

namespace {

// Each thread streams 16-byte words with UNROLL independent loads in flight,
// grid-stride over the buffer, and folds them into one XOR that is written
// out (one atomic per CTA) so the loads cannot be removed.
template <int UNROLL>
__global__ void __launch_bounds__(512) stream_read_kernel(const uint4* __restrict__ src, size_t n16,
                                                         unsigned int* __restrict__ sink) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (UNROLL - 1) * stride < n16; i += UNROLL * stride) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t red[16];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) a ^= red[w];
    atomicXor(sink, a);
  }
}

}  // namespace

extern "C" HQ_API hq_status hq_diag_stream_read(const void* src, size_t bytes, uint32_t* sink, int32_t ctas_per_sm,
                                                hq_stream_t stream) {
  if (src == nullptr || sink == nullptr || (reinterpret_cast<uintptr_t>(src) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(sink) & 3u) != 0 || bytes % 16 != 0 || ctas_per_sm < 1 || ctas_per_sm > 4)
    return HQ_ERR_INVALID;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return hq::cuda_fail(e, "device query");
  stream_read_kernel<4><<<sms * ctas_per_sm, 512, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), bytes / 16, sink);
  return hq::cuda_status(cudaGetLastError(), "stream read launch");
}
