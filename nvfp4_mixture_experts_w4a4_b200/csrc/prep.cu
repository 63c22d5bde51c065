// Weights that arrive already quantised to NVFP4 (E2M1 codes, E4M3 block scales, fp32 tensor
// scales; the SSD-Stream model card's checkpoint stores the routed experts this way, two codes
// per byte) into the layout the layer reads: rows gathered (the gate/up interleave of W13) and
// the block scales moved into the tcgen05 MMA layout, or converted between the two scale
// layouts alone.  A setup step, bytes only: no value is recomputed.
#include <algorithm>

#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr int kPrepThreads = 256;

__device__ __forceinline__ int64_t sf_word_offset(int layout, int64_t r, int64_t g, int64_t K) {
  // byte offset of the four scales of 64-element group g of row r (contiguous in both layouts)
  return layout == NVFP4MOE_SF_MMA ? sf_mma_offset(r, 4 * g, K) : r * (K / 16) + 4 * g;
}

__global__ void prep_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int sf_layout,
                            int64_t batch, int64_t rows, int64_t K, const int32_t* __restrict__ gather,
                            int64_t out_rows, uint8_t* codes_out, uint8_t* sf_out, int out_layout,
                            uint32_t* status) {
  const int64_t groups = K / 64, per = out_rows * groups;
  const int64_t in_sf = sf_layout == NVFP4MOE_SF_MMA ? sf_mma_bytes(rows, K) : rows * (K / 16);
  const int64_t out_sf = out_layout == NVFP4MOE_SF_MMA ? sf_mma_bytes(out_rows, K) : out_rows * (K / 16);
  for (int64_t i = blockIdx.x * int64_t(kPrepThreads) + threadIdx.x; i < batch * per;
       i += int64_t(gridDim.x) * kPrepThreads) {
    const int64_t b = i / per, rg = i - b * per, r = rg / groups, g = rg - r * groups;
    const int64_t src = gather ? gather[r] : r;
    if (src < 0) continue;  // a row another call fills
    if (src >= rows) {      // past the input: skipped and reported
      atomicOr(status, uint32_t(NVFP4MOE_DEV_BAD_GATHER));
      continue;
    }
    const uint32_t w = *reinterpret_cast<const uint32_t*>(sf + b * in_sf + sf_word_offset(sf_layout, src, g, K));
    *reinterpret_cast<uint32_t*>(sf_out + b * out_sf + sf_word_offset(out_layout, r, g, K)) = w;
    if (codes_out) {
      const uint4* s = reinterpret_cast<const uint4*>(codes + (b * rows + src) * (K / 2) + g * 32);
      uint4* d = reinterpret_cast<uint4*>(codes_out + (b * out_rows + r) * (K / 2) + g * 32);
      d[0] = s[0];
      d[1] = s[1];
    }
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

nvfp4moe_status nvfp4_prep_weights(const uint8_t* codes, const uint8_t* sf, int32_t sf_layout, int64_t batch,
                                   int64_t rows, int64_t K, const int32_t* row_gather, int64_t out_rows,
                                   uint8_t* codes_out, uint8_t* sf_out, int32_t sf_out_layout,
                                   nvfp4moe_stream_t stream) {
  const char* fn = "nvfp4_prep_weights";
  NVFP4_REQUIRE(batch >= 0 && rows >= 0 && out_rows >= 0, NVFP4MOE_INVALID_ARG, "%s: negative size", fn);
  NVFP4_REQUIRE(K > 0 && K % 64 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: K=%lld must be a multiple of 64", fn,
                (long long)K);
  auto layout_ok = [](int32_t l) { return l == NVFP4MOE_SF_ROWMAJOR || l == NVFP4MOE_SF_MMA; };
  NVFP4_REQUIRE(layout_ok(sf_layout) && layout_ok(sf_out_layout), NVFP4MOE_INVALID_ARG, "%s: unknown sf layout",
                fn);
  NVFP4_REQUIRE(row_gather != nullptr || out_rows == rows, NVFP4MOE_INVALID_ARG, "%s: out_rows != rows without a gather",
                fn);
  if (batch == 0 || out_rows == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(sf && sf_out, NVFP4MOE_INVALID_ARG, "%s: NULL scale pointer", fn);
  NVFP4_REQUIRE(codes_out == nullptr || codes != nullptr, NVFP4MOE_INVALID_ARG, "%s: codes_out without codes", fn);
  NVFP4_REQUIRE(codes_out == nullptr || (aligned16(codes) && aligned16(codes_out)), NVFP4MOE_INVALID_ARG,
                "%s: codes must be 16-byte aligned", fn);
  NVFP4_REQUIRE((reinterpret_cast<uintptr_t>(sf) & 3u) == 0 && (reinterpret_cast<uintptr_t>(sf_out) & 3u) == 0,
                NVFP4MOE_INVALID_ARG, "%s: scales must be 4-byte aligned", fn);
  uint32_t* status = device_status_ptr();
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_CUDA_ERROR, "%s: device status word unavailable", fn);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = batch * out_rows * (K / 64);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n + kPrepThreads - 1) / kPrepThreads,
                                                                int64_t(num_sms()) * 8));
  prep_kernel<<<grid, kPrepThreads, 0, s>>>(codes, sf, sf_layout, batch, rows, K, row_gather, out_rows, codes_out,
                                            sf_out, sf_out_layout, status);
  return check_launch(fn);
}

}  // extern "C"
