// Two measurement and self-test kernels that sit beside the layer:
//
// nvfp4moe_mma_peak_probe: the ceiling of the block-scaled FP4 tensor-core MMA on this
//   device.  One CTA per SM keeps its operands resident in shared memory (a 128-row weight
//   tile and a 256-row token tile of E2M1 codes, E4M3 block scales staged once into TMEM)
//   and issues `iters` x 4 back-to-back tcgen05.mma kind::mxf4nvf4 (M=128, N=256, K=64) into
//   one TMEM accumulator, with commits every 64 MMAs so at most two batches are in flight.
//   Nothing is loaded from global memory inside the loop, so the launch time is the MMA
//   pipe's: 2*128*256*64 FLOP per MMA.  It is the FP4 roofline denominator of the benchmark.
//
// nvfp4moe_wait_selftest: the bounded-wait path every tcgen05 kernel of the library takes
//   when an mbarrier phase never completes.  One thread waits, with the same mbar_wait as the
//   GEMMs but a caller-given poll limit, on a barrier that nothing ever arrives on; when the
//   limit runs out it sets NVFP4MOE_DEV_TIMEOUT in the device status word and returns.  No
//   fault, trap or hang is involved: the context stays usable.
#include "tcgen05.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int PM = 128, PN = 256;
constexpr int P_A_BYTES = PM * 128;     // K = 256 per row (128 bytes), 128-byte swizzle
constexpr int P_B_BYTES = PN * 128;
constexpr int P_SFA_BYTES = 4 * 512;    // 4 atoms (one per 64 elements of K)
constexpr int P_SFB_BYTES = 2 * 4 * 512;  // two 128-row atom rows
constexpr int P_SMEM = 1024 + P_A_BYTES + P_B_BYTES + P_SFA_BYTES + P_SFB_BYTES + 64;
constexpr int P_SMEM_LAUNCH = 120 * 1024;  // one CTA per SM
constexpr uint32_t P_SFA_COL = PN, P_SFB_COL = PN + 16;
constexpr uint32_t kDevTimeout = NVFP4MOE_DEV_TIMEOUT;

__device__ __forceinline__ uint32_t mix32(uint32_t v) {
  v ^= v >> 16;
  v *= 0x7feb352du;
  v ^= v >> 15;
  v *= 0x846ca68bu;
  v ^= v >> 16;
  return v;
}

__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int64_t iters, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + P_A_BYTES;
  uint8_t* sSFA = sB + P_B_BYTES;
  uint8_t* sSFB = sSFA + P_SFA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + P_SFB_BYTES);  // [2] batches, [1] drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3);
  const int warp = threadIdx.x >> 5;

  // operands: pseudo-random E2M1 codes; block scales 0x20 (2^-3) so sums stay finite
  uint32_t* codes = reinterpret_cast<uint32_t*>(sA);
  for (int i = threadIdx.x; i < (P_A_BYTES + P_B_BYTES) / 4; i += blockDim.x) codes[i] = mix32(i * 2654435761u + 17u);
  uint32_t* sf = reinterpret_cast<uint32_t*>(sSFA);
  for (int i = threadIdx.x; i < (P_SFA_BYTES + P_SFB_BYTES) / 4; i += blockDim.x) sf[i] = 0x20202020u;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 3; ++b) mbar_init(&bars[b], 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  fence_proxy_async_shared();  // the generic stores above, before the tensor core reads them
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 1 && elect_one()) {
    const uint64_t sfa_d = desc_sf_atom(sSFA), sfb_d = desc_sf_atom(sSFB);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tc_cp_sf(tmem + P_SFA_COL + 4 * j, sfa_d + 32 * j);
      tc_cp_sf(tmem + P_SFB_COL + 8 * j, sfb_d + 32 * j);
      tc_cp_sf(tmem + P_SFB_COL + 8 * j + 4, sfb_d + 128 + 32 * j);
    }
    const uint64_t a_d = desc_kmajor_sw128(sA), b_d = desc_kmajor_sw128(sB);
    const uint32_t idesc = idesc_mxf4nvf4(PM, PN);
    bool ok = true;
    for (int64_t it = 0; it < iters && ok; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tc_mma_mxf4nvf4(tmem, a_d + 2 * j, b_d + 2 * j, idesc, tmem + P_SFA_COL + 4 * j, tmem + P_SFB_COL + 8 * j,
                        (it | j) != 0 ? 1u : 0u);
      if ((it & 15) == 15) {
        const int64_t b = it >> 4;
        tc_commit(&bars[b & 1]);
        if (b >= 1 && !mbar_wait(&bars[(b - 1) & 1], uint32_t(((b - 1) >> 1) & 1), 1u << 24)) {
          atomicOr(status, kDevTimeout);
          ok = false;
        }
      }
    }
    tc_commit(&bars[2]);  // every MMA issued above has completed once this arrives
    if (!mbar_wait(&bars[2], 0, 1u << 26)) atomicOr(status, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

__global__ void wait_selftest_kernel(uint32_t polls, uint32_t* status, int32_t* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing arrives on `bar`: its phase 0 never completes
    const bool done = mbar_wait(&bar, 0, polls);
    if (!done) atomicOr(status, kDevTimeout);
    *result = done ? 1 : 0;
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

nvfp4moe_status nvfp4moe_mma_peak_probe(int64_t iters, nvfp4moe_stream_t stream) {
  NVFP4_REQUIRE(iters >= 1 && iters <= (int64_t(1) << 24), NVFP4MOE_INVALID_ARG,
                "nvfp4moe_mma_peak_probe: iters=%lld outside [1, 2^24]", (long long)iters);
  uint32_t* status = device_status_ptr();
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_CUDA_ERROR, "nvfp4moe_mma_peak_probe: device status word unavailable");
  static_assert(P_SMEM <= P_SMEM_LAUNCH, "probe shared memory");
  const cudaError_t a =
      cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_LAUNCH);
  NVFP4_REQUIRE(a == cudaSuccess, NVFP4MOE_CUDA_ERROR, "nvfp4moe_mma_peak_probe: %s", cudaGetErrorString(a));
  mma_peak_kernel<<<num_sms(), 128, P_SMEM_LAUNCH, reinterpret_cast<cudaStream_t>(stream)>>>(iters, status);
  return check_launch("nvfp4moe_mma_peak_probe");
}

int64_t nvfp4moe_mma_peak_probe_flops(int64_t iters) {
  return int64_t(num_sms()) * iters * 4 * 2 * int64_t(PM) * PN * 64;
}

nvfp4moe_status nvfp4moe_wait_selftest(uint32_t polls, int32_t* result, nvfp4moe_stream_t stream) {
  NVFP4_REQUIRE(result != nullptr, NVFP4MOE_INVALID_ARG, "nvfp4moe_wait_selftest: result is NULL");
  NVFP4_REQUIRE(polls >= 1 && polls <= (1u << 20), NVFP4MOE_INVALID_ARG,
                "nvfp4moe_wait_selftest: polls=%u outside [1, 2^20]", polls);
  uint32_t* status = device_status_ptr();
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_CUDA_ERROR, "nvfp4moe_wait_selftest: device status word unavailable");
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(polls, status, result);
  return check_launch("nvfp4moe_wait_selftest");
}

}  // extern "C"
