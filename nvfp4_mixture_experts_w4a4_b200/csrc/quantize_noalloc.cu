// nvfp4_quantize_dynamic_noalloc: the dynamic-scale quantiser for callers that cannot
// allocate device memory.
//
// The dynamic tensor scale needs a little scratch: one fp32 amax per CTA of the first pass
// (see nvfp4_quantize_workspace_size).  Callers such as plug-ins that live inside a host
// framework which owns the device allocator (and forbids side allocations), or deployments
// that reserve their whole device-memory footprint up front, have no workspace to hand us
// and may not call cudaMalloc.  This variant takes its scratch from a fixed array compiled
// into the library instead: kScratchBytes of device memory that every GPU which loads the
// library holds until the process exits.
//
// The array is shared by every call on a device and keeps the previous call's contents.
// That is harmless here: every partial that is read in a call is first written in the same
// call, so nothing needs clearing.  Two calls whose kernels overlap on the GPU (e.g. on
// two streams without ordering between them) race on the array; order them.
#include <mutex>

#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr size_t kScratchBytes = 64 * 1024;  // 16384 fp32 partial maxima

static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

// Device address of g_noalloc_scratch for the current device, looked up once per device.
// In host code the symbol itself is only a host-side stand-in, never a device address.
nvfp4moe_status scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "nvfp4_quantize_dynamic_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64)
    return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "nvfp4_quantize_dynamic_noalloc: device index %d >= 64", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(NVFP4MOE_CUDA_ERROR, "nvfp4_quantize_dynamic_noalloc: cudaGetSymbolAddress failed: %s",
                  cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return NVFP4MOE_OK;
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4moe_status nvfp4_quantize_dynamic_noalloc(
    const void* x, int32_t x_dtype, int64_t batch, int64_t rows, int64_t K, int64_t ldx,
    int64_t x_batch_stride, const int32_t* row_gather, int64_t out_rows, float* tensor_scale,
    uint8_t* codes, int64_t codes_batch_stride, uint8_t* sf, int64_t sf_batch_stride, int32_t sf_layout,
    nvfp4moe_stream_t stream) {
  const char* fn = "nvfp4_quantize_dynamic_noalloc";
  NVFP4_REQUIRE(batch >= 0 && rows >= 0 && K >= 0, NVFP4MOE_INVALID_ARG, "%s: negative size", fn);
  const size_t need = nvfp4_quantize_workspace_size(batch, rows, K);
  NVFP4_REQUIRE(need <= kScratchBytes, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: this size needs %zu bytes of scratch but the built-in scratch holds %zu bytes "
                "(use nvfp4_quantize with a workspace, or split the batch)",
                fn, need, kScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    nvfp4moe_status st = scratch_address(&scratch);
    if (st != NVFP4MOE_OK) return st;
  }
  return nvfp4_quantize(x, x_dtype, batch, rows, K, ldx, x_batch_stride, row_gather, out_rows,
                        NVFP4MOE_SCALE_DYNAMIC, tensor_scale, codes, codes_batch_stride, sf, sf_batch_stride,
                        sf_layout, scratch, kScratchBytes, stream);
}
