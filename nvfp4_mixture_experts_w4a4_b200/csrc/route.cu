// moe_route: router top-k with softmax over the selected logits.
//
// One warp per token.  Lane l holds logits l, l+32, ... in registers (E <= 1024, so at
// most 32 per lane).  Each of the k rounds is a warp arg-max over 64-bit keys: the high
// word is the logit mapped to an unsigned integer with the same order (after -0 is turned
// into +0, so the two zeros tie), the low word is 0xFFFF - index, so among equal logits the
// lower index has the larger key.  Key 0 marks "no candidate".  Integer compares make the
// selection order exact; the softmax weights are fp32.
#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ uint64_t sort_key(float v, int idx) {
  uint32_t u = __float_as_uint(v + 0.0f);  // -0 + +0 = +0 under round-to-nearest
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (uint64_t(u) << 32) | uint32_t(0xFFFF - idx);
}

__device__ __forceinline__ int key_index(uint64_t key) { return 0xFFFF - int(uint32_t(key) & 0xFFFFu); }

template <int PER_LANE>
__global__ void __launch_bounds__(kWarps * 32)
route_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
             float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* l = logits + int64_t(t) * E;
  float v[PER_LANE];
  uint32_t taken = 0;  // bit i: element lane + 32 i already selected (or absent)
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? l[e] : 0.0f;
    if (e >= E) taken |= 1u << i;
  }
  float sel_v = 0.0f;  // lane j keeps the j-th selected logit
  int sel_i = 0;
  for (int j = 0; j < k; ++j) {
    uint64_t best = 0;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      const uint64_t key = (taken >> i & 1u) ? 0ull : sort_key(v[i], lane + 32 * i);
      best = key > best ? key : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    const int bi = key_index(best);  // the same on every lane
    if ((bi & 31) == lane) {
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i)
        if (i == (bi >> 5)) taken |= 1u << i;
    }
    const float bv = __shfl_sync(0xffffffffu, [&] {
      float r = 0.0f;
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i)
        if (i == (bi >> 5)) r = v[i];
      return r;
    }(), bi & 31);
    if (lane == j) {
      sel_v = bv;
      sel_i = bi;
    }
  }
  // softmax over the k selected logits, relative to the largest (the first)
  const float l0 = __shfl_sync(0xffffffffu, sel_v, 0);
  const float ex = lane < k ? expf(sel_v - l0) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[int64_t(t) * k + lane] = sel_i;
    w[int64_t(t) * k + lane] = ex / sum;
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
