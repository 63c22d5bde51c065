// Error plumbing, the device status word, and the exposed element codec.
#include <cstdarg>
#include <mutex>

#include "common.cuh"

namespace nvfp4moe {

namespace {
thread_local std::string g_last_error;
}

// Sticky fault word, one per device (every device that loads the module has its copy).
__device__ uint32_t g_device_status = 0;

void set_error(const std::string& msg) { g_last_error = msg; }

nvfp4moe_status fail(nvfp4moe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

nvfp4moe_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "%s: %s", what, cudaGetErrorString(e));
  return NVFP4MOE_OK;
}

uint32_t* device_status_ptr() {
  static std::mutex mu;
  static uint32_t* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  return ptrs[dev];
}

namespace {
__global__ void codec_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ e2m1,
                             uint8_t* __restrict__ e4m3) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float v = in[i];
    if (e2m1) e2m1[i] = static_cast<uint8_t>(e2m1x2_from_f32(v, 0.0f) & 0xFu);
    if (e4m3) e4m3[i] = static_cast<uint8_t>(e4m3_from_f32(v));
  }
}
}  // namespace

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

const char* nvfp4moe_last_error(void) { return g_last_error.c_str(); }

int32_t nvfp4moe_version(void) { return 0x000600; }

nvfp4moe_status nvfp4moe_device_status(nvfp4moe_stream_t stream, int32_t clear, uint32_t* status) {
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_INVALID_ARG, "nvfp4moe_device_status: status is NULL");
  uint32_t* p = device_status_ptr();
  NVFP4_REQUIRE(p != nullptr, NVFP4MOE_CUDA_ERROR, "nvfp4moe_device_status: no device symbol");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(status, p, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(p, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  NVFP4_REQUIRE(e == cudaSuccess, NVFP4MOE_CUDA_ERROR, "nvfp4moe_device_status: %s",
                cudaGetErrorString(e));
  return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4_codec_convert(const float* in, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                    nvfp4moe_stream_t stream) {
  NVFP4_REQUIRE(n >= 0, NVFP4MOE_INVALID_ARG, "nvfp4_codec_convert: n < 0");
  if (n == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(in != nullptr, NVFP4MOE_INVALID_ARG, "nvfp4_codec_convert: in is NULL");
  const int threads = 256;
  const int64_t want = (n + threads - 1) / threads;
  const int blocks = static_cast<int>(want < int64_t(num_sms()) * 16 ? want : int64_t(num_sms()) * 16);
  codec_kernel<<<blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, n, e2m1, e4m3);
  return check_launch("nvfp4_codec_convert");
}

}  // extern "C"
