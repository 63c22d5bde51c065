// MXFP4 weights on the NVFP4 kernels.
//
// MXFP4 (E2M1 elements, one E8M0 power-of-two scale per 32 elements along K; the format the
// DwarfStar CUDA multi-GPU doc names as its launcher's default, read as the OCP microscaling
// definition) shares its element codes with NVFP4.  A power of two 2^j is exactly an E4M3
// value for j in [-9, 8], so an MXFP4 matrix has an exact NVFP4 form whenever the scales of
// its nonzero blocks span at most 18 binades: each 16-element half of a block takes the E4M3
// scale 2^(E - 127 - shift), the matrix the tensor scale 2^shift, shift = (largest E of a
// nonzero block) - 135.  The conversion runs once per weight matrix (setup, not the layer's
// hot path) and is synchronous: it reports a matrix without an exact form as an error.
#include <algorithm>
#include <vector>

#include "common.cuh"

namespace nvfp4moe {
namespace {

// 2^j as an fp32 (subnormal below 2^-126; j >= -149)
__device__ __forceinline__ float pow2f(int j) {
  return j >= -126 ? __int_as_float((j + 127) << 23) : __int_as_float(1 << (j + 149));
}

// E4M3 code of 2^j, j in [-9, 8]
__device__ __forceinline__ uint32_t e4m3_pow2(int j) { return j >= -6 ? uint32_t(j + 7) << 3 : 1u << (j + 9); }

__device__ __forceinline__ bool block_nonzero(const uint8_t* codes16) {
  const uint4 v = *reinterpret_cast<const uint4*>(codes16);
  return ((v.x | v.y | v.z | v.w) & 0x77777777u) != 0u;  // any nonzero magnitude nibble
}

// ws[2b] = 1 + largest E8M0 code of a nonzero block of matrix b (0: none)
__global__ void mx_emax_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ e8m0, int64_t batch,
                               int64_t rows, int64_t K, int* ws) {
  const int64_t nb = K / 32, per = rows * nb;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < batch * per; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = i / per, rb = i - b * per, r = rb / nb, k = rb - r * nb;
    const uint8_t* c = codes + (b * rows + r) * (K / 2) + k * 16;
    if (block_nonzero(c)) atomicMax(&ws[2 * b], int(e8m0[(b * rows + r) * nb + k]) + 1);
  }
}

__global__ void mx_convert_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ e8m0, int64_t batch,
                                  int64_t rows, int64_t K, const int32_t* __restrict__ gather, int64_t out_rows,
                                  uint8_t* codes_out, uint8_t* sf_out, float* tensor_scale, int* ws) {
  const int64_t nb = K / 32, per = out_rows * nb;
  const int64_t sf_per = sf_mma_bytes(out_rows, K);
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < batch * per; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = i / per, rb = i - b * per, r = rb / nb, k = rb - r * nb;
    const int emax1 = ws[2 * b];
    const int shift = emax1 > 0 ? emax1 - 1 - 135 : 0;
    if (rb == 0) tensor_scale[b] = pow2f(shift);
    const int64_t src = gather ? gather[r] : r;
    if (src < 0) continue;  // an out row another call fills
    if (src >= rows) {      // a gather entry past the input: flagged, the row left untouched
      atomicOr(&ws[2 * b + 1], 2);
      continue;
    }
    const uint8_t* c = codes + (b * rows + src) * (K / 2) + k * 16;
    uint32_t code = 0u;
    if (block_nonzero(c)) {
      const int j = int(e8m0[(b * rows + src) * nb + k]) - 127 - shift;
      if (j < -9) {
        atomicOr(&ws[2 * b + 1], 1);  // no exact NVFP4 form
      } else {
        code = e4m3_pow2(j);
      }
    }
    uint8_t* sf = sf_out + b * sf_per;
    sf[sf_mma_offset(r, 2 * k, K)] = static_cast<uint8_t>(code);
    sf[sf_mma_offset(r, 2 * k + 1, K)] = static_cast<uint8_t>(code);
    if (codes_out)
      *reinterpret_cast<uint4*>(codes_out + (b * out_rows + r) * (K / 2) + k * 16) = *reinterpret_cast<const uint4*>(c);
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

size_t nvfp4_from_mxfp4_workspace_size(int64_t batch) { return size_t(batch > 0 ? batch : 1) * 8; }

nvfp4moe_status nvfp4_from_mxfp4(const uint8_t* codes, const uint8_t* e8m0, int64_t batch, int64_t rows, int64_t K,
                                 const int32_t* row_gather, int64_t out_rows, uint8_t* codes_out, uint8_t* sf_out,
                                 float* tensor_scale, void* workspace, size_t workspace_bytes,
                                 nvfp4moe_stream_t stream) {
  const char* fn = "nvfp4_from_mxfp4";
  NVFP4_REQUIRE(batch >= 0 && rows >= 0 && out_rows >= 0, NVFP4MOE_INVALID_ARG, "%s: negative size", fn);
  NVFP4_REQUIRE(K > 0 && K % 64 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: K=%lld must be a multiple of 64", fn,
                (long long)K);
  NVFP4_REQUIRE(row_gather != nullptr || out_rows == rows, NVFP4MOE_INVALID_ARG, "%s: out_rows != rows without a gather",
                fn);
  if (batch == 0 || out_rows == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(codes && e8m0 && sf_out && tensor_scale && workspace, NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  NVFP4_REQUIRE(workspace_bytes >= nvfp4_from_mxfp4_workspace_size(batch), NVFP4MOE_WORKSPACE_TOO_SMALL,
                "%s: workspace too small", fn);
  NVFP4_REQUIRE(aligned16(codes) && (codes_out == nullptr || aligned16(codes_out)), NVFP4MOE_INVALID_ARG,
                "%s: codes must be 16-byte aligned", fn);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, size_t(batch) * 8, s);
  NVFP4_REQUIRE(e == cudaSuccess, NVFP4MOE_CUDA_ERROR, "%s: %s", fn, cudaGetErrorString(e));
  const int64_t n1 = batch * rows * (K / 32), n2 = batch * out_rows * (K / 32);
  auto grid = [](int64_t n) { return static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, int64_t(num_sms()) * 8)); };
  if (n1 > 0) mx_emax_kernel<<<grid(n1), 256, 0, s>>>(codes, e8m0, batch, rows, K, ws);
  mx_convert_kernel<<<grid(n2), 256, 0, s>>>(codes, e8m0, batch, rows, K, row_gather, out_rows, codes_out, sf_out,
                                             tensor_scale, ws);
  nvfp4moe_status st = check_launch(fn);
  if (st != NVFP4MOE_OK) return st;
  // synchronous: report matrices without an exact NVFP4 form
  std::string bad;
  {
    std::vector<int> host(size_t(batch) * 2);
    e = cudaMemcpyAsync(host.data(), ws, size_t(batch) * 8, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    NVFP4_REQUIRE(e == cudaSuccess, NVFP4MOE_CUDA_ERROR, "%s: %s", fn, cudaGetErrorString(e));
    for (int64_t b = 0; b < batch && bad.size() < 64; ++b)
      if (host[size_t(2 * b + 1)] & 1) bad += (bad.empty() ? "" : ",") + std::to_string(b);
    for (int64_t b = 0; b < batch; ++b)
      NVFP4_REQUIRE(!(host[size_t(2 * b + 1)] & 2), NVFP4MOE_INVALID_ARG, "%s: row_gather names a row >= rows (%lld)",
                    fn, (long long)rows);
  }
  NVFP4_REQUIRE(bad.empty(), NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: matrices [%s] have nonzero blocks whose scales span more than 18 binades (no exact NVFP4 form)",
                fn, bad.c_str());
  return NVFP4MOE_OK;
}

}  // extern "C"
