// moe_route: router top-k with softmax over the selected logits.
// One warp per token; the selection is warp_topk (topk.cuh).
#include "topk.cuh"

namespace nvfp4moe {
namespace {

constexpr int kWarps = 8;

template <int PER_LANE>
__global__ void __launch_bounds__(kWarps * 32)
route_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
             float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int id;
  float wt;
  warp_topk<PER_LANE>(logits + int64_t(t) * E, E, k, &id, &wt);
  if (lane < k) {
    ids[int64_t(t) * k + lane] = id;
    w[int64_t(t) * k + lane] = wt;
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k,
                                     int32_t* ids, float* w, nvfp4moe_stream_t stream) {
  const char* fn = "moe_route";
  NVFP4_REQUIRE(T >= 0, NVFP4MOE_INVALID_ARG, "%s: T < 0", fn);
  NVFP4_REQUIRE(E >= 1 && E <= 1024, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: E=%d outside [1, 1024]", fn, E);
  NVFP4_REQUIRE(k >= 1 && k <= 32 && k <= E, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: k=%d outside [1, min(E, 32)]", fn, k);
  if (T == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(logits && ids && w, NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int blocks = (T + kWarps - 1) / kWarps;
  const int per = (E + 31) / 32;
  if (per <= 1)
    route_kernel<1><<<blocks, kWarps * 32, 0, s>>>(logits, T, E, k, ids, w);
  else if (per <= 4)
    route_kernel<4><<<blocks, kWarps * 32, 0, s>>>(logits, T, E, k, ids, w);
  else if (per <= 8)
    route_kernel<8><<<blocks, kWarps * 32, 0, s>>>(logits, T, E, k, ids, w);
  else if (per <= 16)
    route_kernel<16><<<blocks, kWarps * 32, 0, s>>>(logits, T, E, k, ids, w);
  else
    route_kernel<32><<<blocks, kWarps * 32, 0, s>>>(logits, T, E, k, ids, w);
  return check_launch(fn);
}
