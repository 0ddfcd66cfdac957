// Measurement aids (declared in include/moe_b200_measure.h): a plain streaming
// read of device memory, the ceiling a read-only weight stream is held to, and
// the TMA weight-panel stream of the grouped GEMMs without their MMAs.
#include "moe_b200_measure.h"
#include "common.cuh"
#include "kernels.h"

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

// ---------------------------------------------------------------------------
// The weight-panel stream of the grouped GEMMs without the GEMM (moe_measure_tma_stream).
namespace {

constexpr int kPanelRows = 128;
constexpr int kPanelCols = 7168;                     // bf16 columns of the panel view
constexpr uint32_t kBox = kPanelRows * 64 * 2;       // one 128 x 64 bf16 box: 16 KB
constexpr int kMaxStages = 16;
constexpr uint32_t kMaxRing = 192 * 1024;

struct TmaStreamArgs {
  const uint8_t* base;
  long long npanels;
  int boxes, stages, contiguous, warps, steps;
  int32_t* err;
};

// Issuer w (lane 0 of warp w) takes the steps i with i % warps == w.  Step i uses slot i % stages; since
// stages is a multiple of warps, step i + stages (the next use of that slot) belongs to the same issuer,
// which issues it only after it has seen step i land, so a slot is never re-armed while its copy is in
// flight and no issuer waits on a phase another issuer has yet to arm.
__global__ void __launch_bounds__(128, 1) tma_stream_kernel(const __grid_constant__ CUtensorMap map, TmaStreamArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kMaxStages];
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) moe::mbar_init(&full[s], 1);
    moe::fence_mbar_init();
  }
  __syncthreads();
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) != 0 || w >= a.warps) return;  // one thread per issuing warp, as the GEMMs' producers
  constexpr int nk = kPanelCols / 64;
  const uint32_t stage_bytes = kBox * static_cast<uint32_t>(a.boxes);
  // first row of box b's panel at step i: this CTA's sequence of panels, box b offset by half the panels
  auto panel_row = [&](int i, int b) -> int {
    const long long pi = static_cast<long long>(blockIdx.x) + static_cast<long long>(i / nk) * gridDim.x;
    return static_cast<int>(((pi * 7919 + b * (a.npanels / 2)) % a.npanels) * kPanelRows);
  };
  auto issue = [&](int i) {
    const int s = i % a.stages, k = i % nk;
    moe::mbar_arrive_expect_tx(&full[s], stage_bytes);
    for (int b = 0; b < a.boxes; ++b) {
      uint8_t* dst = ring + static_cast<size_t>(s) * stage_bytes + b * kBox;
      const int row = panel_row(i, b);
      if (a.contiguous)  // the panel stored box by box: box k is bytes [k * 16 KB, (k + 1) * 16 KB) of the panel
        moe::bulk_load(dst, a.base + static_cast<size_t>(row) * (kPanelCols * 2) + static_cast<size_t>(k) * kBox, kBox,
                       &full[s]);
      else
        moe::tma_load_2d(&map, &full[s], dst, k * 64, row);
    }
  };
  for (int i = w; i < a.stages && i < a.steps; i += a.warps) issue(i);
  for (int i = w; i < a.steps; i += a.warps) {
    const int s = i % a.stages;
    if (!moe::mbar_wait_bounded(&full[s], (i / a.stages) & 1, nullptr)) {
      moe::set_error(a.err, moe::kErrTimeout);
      // this issuer's copies still in flight land before it leaves
      for (int j = i + a.warps; j < i + a.stages && j < a.steps; j += a.warps)
        moe::mbar_wait_bounded(&full[j % a.stages], (j / a.stages) & 1, nullptr);
      return;
    }
    if (i + a.stages < a.steps) issue(i + a.stages);
  }
}

}  // namespace

extern "C" moe_status_t moe_measure_tma_stream(const void* buf, size_t bytes, int boxes, int stages, int contiguous,
                                               int warps, int steps, int32_t* err, size_t* bytes_moved,
                                               moe_stream_t stream) {
  const size_t row_bytes = static_cast<size_t>(kPanelCols) * 2;
  const size_t rows = bytes / row_bytes;
  if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || rows < kPanelRows) return MOE_ERR_INVALID_ARG;
  if (boxes < 1 || boxes > 3 || stages < 2 || stages > kMaxStages || steps < 1) return MOE_ERR_INVALID_ARG;
  if (warps < 1 || warps > 4 || stages % warps != 0) return MOE_ERR_INVALID_ARG;
  const uint32_t ring = kBox * static_cast<uint32_t>(boxes * stages);
  if (ring > kMaxRing) return MOE_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return MOE_ERR_CUDA;
  CUtensorMap map;
  if (!moe::encode_map_bf16(&map, buf, rows, kPanelCols, kPanelRows)) return MOE_ERR_CUDA;
  const size_t smem = ring + 1024;
  if (cudaFuncSetAttribute(tma_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  TmaStreamArgs a{static_cast<const uint8_t*>(buf), static_cast<long long>(rows / kPanelRows), boxes, stages,
                  contiguous != 0, warps, steps, err};
  tma_stream_kernel<<<sms, 32 * warps, smem, static_cast<cudaStream_t>(stream)>>>(map, a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (bytes_moved != nullptr) *bytes_moved = static_cast<size_t>(sms) * steps * boxes * kBox;
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// The copy mix of the NVFP4 GEMMs' stages without the GEMM (moe_measure_tma_mix).
namespace {

constexpr int kMixRowBytes = 3584;                    // e2m1 codes of a 7168-element row
constexpr int kMixTokenRows = 8192;                   // token rows: the first 28 MB, resident in L2
constexpr uint32_t kMixCodeBox = 128 * 128;           // 128 rows x 128 bytes
constexpr uint32_t kMixTokenBox = 64 * 128;           // 64 rows x 128 bytes
constexpr uint32_t kMixSf = 2048, kMixSf4 = 8192;     // scales of one k-step / of four
constexpr uint32_t kMixSfRing = 2 * 3 * kMixSf4;      // mix 4: two groups of three 8 KB chunks

// Bytes of one ring slot: the code boxes, the token box and (mixes 2 and 3) one step's scales.
__host__ __device__ constexpr uint32_t mix_slot_bytes(int mix) {
  return 2 * kMixCodeBox + (mix >= 1 ? kMixTokenBox : 0) + ((mix == 2 || mix == 3) ? 3 * kMixSf : 0);
}

struct TmaMixArgs {
  int mix, stages, steps;
  long long npanels, sf_chunks4;  // panels of codes; 8 KB scale chunks
  int32_t* err;
};

__device__ __forceinline__ uint32_t mix_step_bytes(int mix, int i) {
  uint32_t b = 2 * kMixCodeBox;
  if (mix >= 1) b += kMixTokenBox;
  if (mix == 2 || mix == 3) b += 3 * kMixSf;
  if (mix == 4 && i % 4 == 0) b += 3 * kMixSf4;
  return b;
}

// Lane 0 of warps 0 and 1 issue; each waits for the slot's previous step to land before refilling it, and warp 0
// posts the step's bytes (the second warp's copies may land first: the barrier's pending arrival holds the phase).
__global__ void __launch_bounds__(64, 1) tma_mix_kernel(const __grid_constant__ CUtensorMap codes,
                                                        const __grid_constant__ CUtensorMap tokens,
                                                        const __grid_constant__ CUtensorMap sf, TmaMixArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t slot = mix_slot_bytes(a.mix);
  uint8_t* sf_ring = ring + static_cast<size_t>(a.stages) * slot;
  __shared__ __align__(8) uint64_t full[4];
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) moe::mbar_init(&full[s], 1);
    moe::fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) != 0) return;
  if (warp == 1 && a.mix == 0) return;
  constexpr int nk = kMixRowBytes / 128;
  auto issue = [&](int i) {
    const int s = i % a.stages, k = i % nk;
    const long long pi = static_cast<long long>(blockIdx.x) + static_cast<long long>(i / nk) * gridDim.x;
    const long long panel = (pi * 7919) % a.npanels;
    uint8_t* st = ring + static_cast<size_t>(s) * slot;
    const long long chunk = (panel * nk + k) * 3;  // this step's three 2 KB scale chunks
    if (warp == 0) {
      moe::mbar_arrive_expect_tx(&full[s], mix_step_bytes(a.mix, i));
      for (int b = 0; b < 2; ++b) {
        const int row = static_cast<int>(((panel + b * (a.npanels / 2)) % a.npanels) * 128);
        moe::tma_load_2d(&codes, &full[s], st + b * kMixCodeBox, k * 128, row);
      }
      if (a.mix == 3)
        moe::tma_load_2d(&sf, &full[s], st + 2 * kMixCodeBox + kMixTokenBox, 0,
                         static_cast<int>((chunk % (a.sf_chunks4 * 4)) * (kMixSf / 256)));
    } else {
      const int trow = static_cast<int>((pi % (kMixTokenRows / 64)) * 64);
      moe::tma_load_2d(&tokens, &full[s], st + 2 * kMixCodeBox, k * 128, trow);
      if (a.mix == 2 || a.mix == 3) {
        for (int j = a.mix == 3 ? 1 : 0; j < 3; ++j)
          moe::tma_load_2d(&sf, &full[s], st + 2 * kMixCodeBox + kMixTokenBox + j * kMixSf, 0,
                           static_cast<int>(((chunk + j) % (a.sf_chunks4 * 4)) * (kMixSf / 256)));
      } else if (a.mix == 4 && i % 4 == 0) {
        uint8_t* dst = sf_ring + static_cast<size_t>((i / 4) % 2) * 3 * kMixSf4;
        for (int j = 0; j < 3; ++j)
          moe::tma_load_2d(&sf, &full[s], dst + j * kMixSf4, 0,
                           static_cast<int>(((chunk / 12 * 3 + j) % a.sf_chunks4) * (kMixSf4 / 256)));
      }
    }
  };
  for (int i = 0; i < a.stages && i < a.steps; ++i) issue(i);
  for (int i = 0; i < a.steps; ++i) {
    const int s = i % a.stages;
    if (!moe::mbar_wait_bounded(&full[s], (i / a.stages) & 1, nullptr)) {
      moe::set_error(a.err, moe::kErrTimeout);
      for (int j = i + 1; j < i + a.stages && j < a.steps; ++j)
        moe::mbar_wait_bounded(&full[j % a.stages], (j / a.stages) & 1, nullptr);
      return;
    }
    if (i + a.stages < a.steps) issue(i + a.stages);
  }
}

}  // namespace

extern "C" moe_status_t moe_measure_tma_mix(const void* buf, size_t bytes, int mix, int stages, int steps, int32_t* err,
                                            size_t* bytes_moved, moe_stream_t stream) {
  if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || bytes < (size_t(256) << 20))
    return MOE_ERR_INVALID_ARG;
  if (mix < 0 || mix > 4 || stages < 2 || stages > 4 || steps < 8) return MOE_ERR_INVALID_ARG;
  const size_t sf_bytes = (bytes / 8) & ~size_t(kMixSf4 - 1);
  const size_t code_bytes = (bytes - sf_bytes) & ~size_t(kMixSf4 - 1);
  const size_t rows = code_bytes / kMixRowBytes;
  const uint8_t* sf_base = static_cast<const uint8_t*>(buf) + code_bytes;  // 16-byte aligned: code_bytes % 8192 == 0
  CUtensorMap codes, tokens, sf;
  if (!moe::encode_map_u8(&codes, buf, rows, kMixRowBytes, 128) ||
      !moe::encode_map_u8(&tokens, buf, kMixTokenRows, kMixRowBytes, 64) ||
      !moe::encode_map_sf_rows(&sf, sf_base, sf_bytes, mix == 4 ? kMixSf4 / 256 : kMixSf / 256))
    return MOE_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return MOE_ERR_CUDA;
  const size_t smem = static_cast<size_t>(stages) * mix_slot_bytes(mix) + (mix == 4 ? kMixSfRing : 0) + 1024;
  if (cudaFuncSetAttribute(tma_mix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  TmaMixArgs a{mix, stages, steps, static_cast<long long>(rows / 128), static_cast<long long>(sf_bytes / kMixSf4), err};
  tma_mix_kernel<<<sms, 64, smem, static_cast<cudaStream_t>(stream)>>>(codes, tokens, sf, a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (bytes_moved != nullptr) {
    double per = 2.0 * kMixCodeBox;
    if (mix >= 1) per += kMixTokenBox;
    if (mix == 2 || mix == 3) per += 3.0 * kMixSf;
    if (mix == 4) per += 3.0 * kMixSf4 / 4;
    *bytes_moved = static_cast<size_t>(per * sms * steps);
  }
  return MOE_OK;
}
