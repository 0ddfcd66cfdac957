// Measurement aid (declared in include/moe_b200_measure.h): a plain streaming
// read of device memory, the ceiling a read-only weight stream is held to.
#include "moe_b200_measure.h"
#include "common.cuh"

namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 4;
constexpr int kInFlight = 8;

__device__ __forceinline__ uint4 ld_nc_16(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kThreads) hbm_read_kernel(const uint4* __restrict__ p, size_t n,
                                                           uint32_t* __restrict__ sink) {
  const size_t stride = static_cast<size_t>(gridDim.x) * kThreads;
  size_t i = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (kInFlight - 1) * stride < n; i += kInFlight * stride) {
    uint4 v[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) v[u] = ld_nc_16(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n; i += stride) {
    const uint4 v = ld_nc_16(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (acc == 0xFFFFFFFFu && sink != nullptr) atomicOr(sink, 1u);
}

}  // namespace

extern "C" moe_status_t moe_measure_hbm_read(const void* buf, size_t bytes, uint32_t* sink, moe_stream_t stream) {
  if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || bytes % 16 != 0 || bytes == 0)
    return MOE_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return MOE_ERR_CUDA;
  hbm_read_kernel<<<sms * kCtasPerSm, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(buf), bytes / 16, sink);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
