// Shared device helpers of libnvfp4moe: NVFP4 element codec, block-scale layout, and the
// status / error plumbing of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/nvfp4moe.h"

namespace nvfp4moe {

// ------------------------------------------------------------------ errors ----
void set_error(const std::string& msg);
nvfp4moe_status fail(nvfp4moe_status st, const char* fmt, ...);
nvfp4moe_status check_launch(const char* what);
uint32_t* device_status_ptr();  // sticky fault word of the current device (nullptr on error)

#define NVFP4_REQUIRE(cond, st, ...) \
  do {                               \
    if (!(cond)) return ::nvfp4moe::fail((st), __VA_ARGS__); \
  } while (0)

inline int num_sms() {
  static std::atomic<int> sms[64];  // zero-initialised (static storage); 0 = not read yet
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  int v = sms[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 148;
    sms[dev].store(v, std::memory_order_relaxed);  // every thread computes the same value
  }
  return v;
}

// Raises kernel Kern's dynamic shared-memory limit to `bytes` on the current device, once per
// device and thread-safe.  A failed attempt is returned and retried by the next call.
template <auto Kern>
cudaError_t set_smem_limit_once(int bytes) {
  static std::mutex mu;
  static int done[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
  return e;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------- programmatic dependent launch ----
// A kernel launched with launch_dependent() may start while the previous kernel on the stream
// is still running: it must call griddep_wait() before touching that kernel's output, and
// griddep_wait() returns once the previous grid has completed and its writes are visible.
// griddep_launch_dependents() lets the next such launch start early (its blocks still only
// get SMs that are free).  Both are no-ops for kernels launched the ordinary way.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Records a timing mark on stream s.  Under stream capture the record must be an external
// event node to stay a timing point of the graph; outside capture that flag is not allowed.
inline cudaError_t record_mark(void* event, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  cudaEvent_t ev = static_cast<cudaEvent_t>(event);
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                              : cudaEventRecord(ev, s);
}

// As launch_dependent, and cooperative: the launch fails unless every block of the grid can be
// resident at once (kernels whose blocks wait on one another).
template <typename... KArgs, typename... Args>
cudaError_t launch_cooperative_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------- element codec ----
// Two fp32 -> two E2M1 codes, round to nearest even, saturating (hardware cvt).
// Returns a byte with `lo` in bits 0..3 and `hi` in bits 4..7.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// Two fp32 -> two E4M3 bytes (round to nearest even, saturate to +-448); lo in bits 0..7.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
  return out;
}

__device__ __forceinline__ uint32_t e4m3_from_f32(float v) { return e4m3x2_from_f32(v, 0.f) & 0xFFu; }

// Two E4M3 bytes (low 16 bits of v) -> f16x2 (exact).
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint32_t v) {
  uint32_t out;
  uint16_t in = static_cast<uint16_t>(v);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(in));
  return out;
}

__device__ __forceinline__ float f32_from_e4m3(uint32_t byte) {
  const uint32_t h2 = f16x2_from_e4m3x2(byte & 0xFFu);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Four E2M1 codes (two bytes, low 16 bits of v) -> two f16x2 (exact):
// out[0] = {elem0, elem1}, out[1] = {elem2, elem3} (low half = lower element).
__device__ __forceinline__ void f16x2x2_from_e2m1x4(uint32_t v, uint32_t& o0, uint32_t& o1) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t}"
      : "=r"(o0), "=r"(o1)
      : "r"(v));
}

// Eight E2M1 codes (one 32-bit word) -> four f16x2.
__device__ __forceinline__ void f16x2x4_from_e2m1x8(uint32_t v, uint32_t o[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(v));
}

// ------------------------------------------------------ block-scale layout ----
// Byte offset of the scale of (row r, 16-element block b) in the MMA layout of a
// matrix with K columns (K % 64 == 0): 128-row x 64-column atoms of 512 bytes, atoms
// contiguous along K; inside an atom row r sits at (r%32)*16 + ((r%128)/32)*4 + b%4.
__host__ __device__ __forceinline__ int64_t sf_mma_offset(int64_t r, int64_t b, int64_t K) {
  return ((r >> 7) * (K >> 6) + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

__host__ __device__ __forceinline__ int64_t sf_mma_bytes(int64_t rows, int64_t K) {
  return ((rows + 127) / 128) * 128 * (K / 16);
}

// ------------------------------------------------------ the block quantiser ----
// Scale of one 16-element block with amax `amax` under tensor scale `s_t`.
// Returns the E4M3 code; writes the fp32 reciprocal element scale to *inv (0 when the
// block scale is zero, meaning every code of the block is zero).
__device__ __forceinline__ uint32_t block_scale(float amax, float s_t, float* inv) {
  if (s_t == 0.0f) {
    *inv = 0.0f;
    return 0u;
  }
  const float ratio = __fdiv_rn(amax, __fmul_rn(6.0f, s_t));
  const uint32_t sf = e4m3_from_f32(ratio);
  const float sfv = f32_from_e4m3(sf);
  *inv = (sfv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sfv, s_t));
  return sf;
}

// Encodes 16 fp32 values (one block) with reciprocal scale inv into 8 bytes (2 words).
__device__ __forceinline__ uint2 encode_block16(const float* v, float inv) {
  uint32_t w[2] = {0u, 0u};
  if (inv != 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = e2m1x2_from_f32(__fmul_rn(v[2 * i], inv), __fmul_rn(v[2 * i + 1], inv));
      w[i >> 2] |= byte << (8 * (i & 3));
    }
  }
  return make_uint2(w[0], w[1]);
}

}  // namespace nvfp4moe
