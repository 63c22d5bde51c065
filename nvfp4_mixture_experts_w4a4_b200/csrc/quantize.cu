// nvfp4_quantize: bf16 / fp32 -> NVFP4 codes + E4M3 block scales.
//
// Memory-bound.  One thread quantises one 64-element group of one output row (four
// 16-element blocks): 128-bit loads of the input, 8-byte code stores and one 32-bit scale
// store in the MMA layout (four consecutive blocks of a row are four consecutive bytes
// there).  A dynamic tensor scale takes a first pass that writes one amax per CTA to the
// workspace; the quantising pass reduces those partials at CTA start, so no atomics and
// no zeroing are needed and the result does not depend on scheduling.
#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxAmaxBlocks = 512;

__host__ __device__ inline int amax_blocks_per_item(int64_t rows, int64_t K) {
  const int64_t chunks = rows * (K / 8);
  int64_t b = (chunks + int64_t(kThreads) * 8 - 1) / (int64_t(kThreads) * 8);
  if (b < 1) b = 1;
  if (b > kMaxAmaxBlocks) b = kMaxAmaxBlocks;
  return static_cast<int>(b);
}

template <typename T>
__device__ __forceinline__ void load8(const T* p, float v[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float v[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
amax_kernel(const T* __restrict__ x, int64_t rows, int64_t K, int64_t ldx, int64_t bstride,
            float* __restrict__ partials) {
  const int b = blockIdx.y;
  const T* xb = x + b * bstride;
  const int64_t cpr = K / 8;
  const int64_t chunks = rows * cpr;
  float m = 0.0f;
  for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < chunks;
       i += int64_t(gridDim.x) * kThreads) {
    const int64_t r = i / cpr, c = i - r * cpr;
    float v[8];
    load8<T>(xb + r * ldx + c * 8, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f;
    for (int w = 0; w < kThreads / 32; ++w) t = fmaxf(t, red[w]);
    partials[int64_t(b) * gridDim.x + blockIdx.x] = t;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const T* __restrict__ x, int64_t rows, int64_t K, int64_t ldx, int64_t bstride,
                const int32_t* __restrict__ gather, int64_t out_rows, int dynamic,
                float* __restrict__ tensor_scale, const float* __restrict__ partials, int nparts,
                uint8_t* __restrict__ codes, int64_t cstride, uint8_t* __restrict__ sf,
                int64_t sstride, int sf_mma) {
  const int b = blockIdx.y;
  __shared__ float s_scale;
  if (threadIdx.x == 0) {
    float s_t;
    if (dynamic) {
      float m = 0.0f;
      for (int i = 0; i < nparts; ++i) m = fmaxf(m, partials[int64_t(b) * nparts + i]);
      s_t = __fdiv_rn(m, 2688.0f);
      if (blockIdx.x == 0) tensor_scale[b] = s_t;
    } else {
      s_t = tensor_scale[b];
    }
    s_scale = s_t;
  }
  __syncthreads();
  const float s_t = s_scale;

  const int64_t groups = (K + 63) / 64;  // 64-element groups per row
  const int64_t nblk_row = K / 16;
  const int64_t total = out_rows * groups;
  const T* xb = x + b * bstride;
  uint8_t* cb = codes + b * cstride;
  uint8_t* sb = sf + b * sstride;
  for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * kThreads) {
    const int64_t r = i / groups, g = i - r * groups;
    const int64_t src = gather ? gather[r] : r;
    if (src < 0 || src >= rows) continue;
    const T* xr = xb + src * ldx + g * 64;
    const int nblk = static_cast<int>((nblk_row - g * 4) < 4 ? (nblk_row - g * 4) : 4);
    uint32_t sfword = 0;
    for (int blk = 0; blk < nblk; ++blk) {
      float v[16];
      load8<T>(xr + blk * 16, v);
      load8<T>(xr + blk * 16 + 8, v + 8);
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
      float inv;
      const uint32_t s = block_scale(amax, s_t, &inv);
      const uint2 w = encode_block16(v, inv);
      *reinterpret_cast<uint2*>(cb + r * (K / 2) + (g * 4 + blk) * 8) = w;
      sfword |= s << (8 * blk);
    }
    if (sf_mma) {
      *reinterpret_cast<uint32_t*>(sb + sf_mma_offset(r, g * 4, K)) = sfword;
    } else {
      for (int blk = 0; blk < nblk; ++blk)
        sb[r * nblk_row + g * 4 + blk] = static_cast<uint8_t>(sfword >> (8 * blk));
    }
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

size_t nvfp4_quantize_workspace_size(int64_t batch, int64_t rows, int64_t K) {
  if (batch <= 0 || rows <= 0 || K <= 0) return 0;
  return size_t(batch) * size_t(amax_blocks_per_item(rows, K)) * sizeof(float);
}

nvfp4moe_status nvfp4_quantize(const void* x, int32_t x_dtype, int64_t batch, int64_t rows,
                               int64_t K, int64_t ldx, int64_t x_batch_stride,
                               const int32_t* row_gather, int64_t out_rows, int32_t scale_mode,
                               float* tensor_scale, uint8_t* codes, int64_t codes_batch_stride,
                               uint8_t* sf, int64_t sf_batch_stride, int32_t sf_layout,
                               void* workspace, size_t workspace_bytes,
                               nvfp4moe_stream_t stream) {
  const char* fn = "nvfp4_quantize";
  NVFP4_REQUIRE(x_dtype == NVFP4MOE_DTYPE_BF16 || x_dtype == NVFP4MOE_DTYPE_F32,
                NVFP4MOE_INVALID_ARG, "%s: bad x_dtype %d", fn, x_dtype);
  NVFP4_REQUIRE(scale_mode == NVFP4MOE_SCALE_GIVEN || scale_mode == NVFP4MOE_SCALE_DYNAMIC,
                NVFP4MOE_INVALID_ARG, "%s: bad scale_mode %d", fn, scale_mode);
  NVFP4_REQUIRE(sf_layout == NVFP4MOE_SF_ROWMAJOR || sf_layout == NVFP4MOE_SF_MMA,
                NVFP4MOE_INVALID_ARG, "%s: bad sf_layout %d", fn, sf_layout);
  NVFP4_REQUIRE(batch >= 0 && rows >= 0 && K >= 0 && out_rows >= 0, NVFP4MOE_INVALID_ARG,
                "%s: negative size", fn);
  NVFP4_REQUIRE(batch <= 65535, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: batch > 65535", fn);
  NVFP4_REQUIRE(K % 16 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: K=%lld is not a multiple of 16", fn,
                (long long)K);
  NVFP4_REQUIRE(sf_layout != NVFP4MOE_SF_MMA || K % 64 == 0, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: the MMA scale layout needs K %% 64 == 0 (K=%lld)", fn, (long long)K);
  NVFP4_REQUIRE(row_gather != nullptr || out_rows == rows, NVFP4MOE_INVALID_ARG,
                "%s: out_rows must equal rows without row_gather", fn);
  if (batch == 0 || out_rows == 0 || K == 0) {
    if (scale_mode == NVFP4MOE_SCALE_DYNAMIC && batch > 0 && rows == 0)
      return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "%s: dynamic scale of an empty matrix", fn);
    return NVFP4MOE_OK;
  }
  const int64_t elt = x_dtype == NVFP4MOE_DTYPE_BF16 ? 2 : 4;
  NVFP4_REQUIRE(x && codes && sf && tensor_scale, NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  const bool multi = batch > 1;
  NVFP4_REQUIRE(aligned16(x) && (ldx * elt) % 16 == 0 && (!multi || (x_batch_stride * elt) % 16 == 0),
                NVFP4MOE_INVALID_ARG, "%s: x, ldx and the batch stride must be 16-byte aligned", fn);
  NVFP4_REQUIRE(ldx >= K, NVFP4MOE_INVALID_ARG, "%s: ldx < K", fn);
  NVFP4_REQUIRE(aligned16(codes) && (!multi || codes_batch_stride % 16 == 0) && aligned16(sf) &&
                    (!multi || sf_batch_stride % 16 == 0),
                NVFP4MOE_INVALID_ARG, "%s: codes / sf and their batch strides must be 16-byte aligned", fn);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nparts = amax_blocks_per_item(rows, K);
  float* partials = nullptr;
  if (scale_mode == NVFP4MOE_SCALE_DYNAMIC) {
    NVFP4_REQUIRE(rows > 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: dynamic scale of an empty matrix", fn);
    const size_t need = nvfp4_quantize_workspace_size(batch, rows, K);
    NVFP4_REQUIRE(workspace != nullptr && workspace_bytes >= need, NVFP4MOE_WORKSPACE_TOO_SMALL,
                  "%s: workspace %zu < %zu bytes", fn, workspace_bytes, need);
    partials = static_cast<float*>(workspace);
    dim3 grid(nparts, static_cast<unsigned>(batch));
    if (x_dtype == NVFP4MOE_DTYPE_BF16)
      amax_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
          static_cast<const __nv_bfloat16*>(x), rows, K, ldx, x_batch_stride, partials);
    else
      amax_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(x), rows, K, ldx,
                                                    x_batch_stride, partials);
    nvfp4moe_status st = check_launch(fn);
    if (st != NVFP4MOE_OK) return st;
  }
  const int64_t work = out_rows * ((K + 63) / 64);
  int64_t blocks = (work + kThreads - 1) / kThreads;
  const int64_t cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(batch));
  const int dyn = scale_mode == NVFP4MOE_SCALE_DYNAMIC;
  const int mma = sf_layout == NVFP4MOE_SF_MMA;
  if (x_dtype == NVFP4MOE_DTYPE_BF16)
    quantize_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), rows, K, ldx, x_batch_stride, row_gather, out_rows,
        dyn, tensor_scale, partials, nparts, codes, codes_batch_stride, sf, sf_batch_stride, mma);
  else
    quantize_kernel<float><<<grid, kThreads, 0, s>>>(
        static_cast<const float*>(x), rows, K, ldx, x_batch_stride, row_gather, out_rows, dyn,
        tensor_scale, partials, nparts, codes, codes_batch_stride, sf, sf_batch_stride, mma);
  return check_launch(fn);
}

}  // extern "C"
