// Decode path of the routed layer (few rows per expert): gate/up GEMV with the fused
// SwiGLU + requantise epilogue, down GEMV writing weighted per-slot rows, and the combine.
// Also the small-M path of nvfp4_gemm.
//
// Work is scheduled per warp: one warp item is 32 weight rows of one active expert (for
// gate/up exactly 16 gate + 16 up rows, i.e. one 16-element block of h, so the SwiGLU and
// the requantisation finish inside the warp).  Warps walk the item list with a grid
// stride; the four warps of a CTA take neighbouring items, which share 128-row scale atoms.
// HBM-bound: every weight byte of the touched experts is read once per group of <= 4
// tokens of that expert.
#include "ffn_gemv.cuh"
#include "gemv.cuh"

namespace nvfp4moe {
namespace {

constexpr int kWarpsPerCta = 4;
// resident CTAs per SM the kernels are compiled for (registers per thread <= 128): the weight
// stream's bytes in flight grow with the warps an SM holds
constexpr int kMinCtas = 4;

// ------------------------------------------------------------- gate / up ----
template <int L, int NT>
__device__ __forceinline__ void gateup_group(const GemvGateUpArgs& a, int e, int64_t item_row0,
                                             int64_t r_first, float sg, float su, float sh,
                                             float (*tots)[4]) {
  constexpr int RP = 32 / L;
  constexpr int GROUPS = 32 / (8 * RP);
  const int lane = threadIdx.x & 31;
  const int64_t H = a.H, I = a.I;
  int64_t arow[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) arow[t] = a.row_token[r_first + t];
  const uint8_t* wc = a.w13_codes + int64_t(e) * 2 * I * (H / 2);
  const uint8_t* wsf = a.w13_sf + int64_t(e) * 2 * I * (H / 16);
#pragma unroll
  for (int G = 0; G < GROUPS; ++G) {
    float tot[8][NT];
    warp_dot8<L, NT>(wc, wsf, item_row0 + G * 8 * RP, 2 * I, a.x_codes, a.x_sf, arow, H, 0, H / 32, tot);
    if (lane % L == 0) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) tots[G * 8 * RP + q * RP + lane / L][t] = tot[q][t];
    }
  }
  __syncwarp();
  const int64_t iblk = item_row0 / 32;  // index of the 16-wide block of h
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float h = 0.0f;
    if (lane < 16) {
      const float g = tots[lane][t] * sg;
      const float u = tots[16 + lane][t] * su;
      h = g / (1.0f + expf(-g)) * u;
    }
    float amax = fabsf(h);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float inv;
    const uint32_t sf = block_scale(amax, sh, &inv);
    const uint32_t code = inv != 0.0f ? (e2m1x2_from_f32(__fmul_rn(h, inv), 0.0f) & 0xFu) : 0u;
    const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
    const int64_t prow = r_first + t;
    if (lane < 16 && (lane & 1) == 0)
      a.h_codes[prow * (I / 2) + iblk * 8 + lane / 2] = static_cast<uint8_t>(code | (hi << 4));
    if (lane == 0) {
      a.h_sf[sf_mma_offset(prow, iblk, I)] = static_cast<uint8_t>(sf);
      if (a.h_amax) atomicMax(reinterpret_cast<int*>(a.h_amax + e), __float_as_int(amax));
    }
  }
  __syncwarp();
}

template <int L>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kMinCtas) gemv_gateup_kernel(GemvGateUpArgs a) {
  __shared__ float tots_all[kWarpsPerCta][32][4];
  const int warp = threadIdx.x >> 5;
  float(*tots)[4] = tots_all[warp];
  const int64_t per_expert = (2 * int64_t(a.I)) / 32;
  const int64_t n_items = int64_t(a.active[0]) * per_expert;
  const float s_x = *a.x_scale;
  for (int64_t item = int64_t(blockIdx.x) * kWarpsPerCta + warp; item < n_items;
       item += int64_t(gridDim.x) * kWarpsPerCta) {
    const int e = a.active[1 + item / per_expert];
    const int64_t row0 = (item % per_expert) * 32;
    const int64_t r0 = a.offsets[e], n_e = a.offsets[e + 1] - r0;
    const float sg = a.w13_scale[2 * e] * s_x, su = a.w13_scale[2 * e + 1] * s_x;
    const float sh = a.h_scale[e];
    int64_t g = 0;
    for (; g + 2 <= n_e; g += 2) gateup_group<L, 2>(a, e, row0, r0 + g, sg, su, sh, tots);
    if (g < n_e) gateup_group<L, 1>(a, e, row0, r0 + g, sg, su, sh, tots);
  }
}

// ------------------------------------------------------------------ down ----
template <int L, int NT>
__device__ __forceinline__ void down_group(const GemvDownArgs& a, int e, int64_t item_row0,
                                           int64_t r_first, int64_t c0, int64_t c1, float sc,
                                           float* slots) {
  constexpr int RP = 32 / L;
  constexpr int GROUPS = 32 / (8 * RP);
  const int lane = threadIdx.x & 31;
  const int64_t H = a.H, I = a.I;
  int64_t arow[NT];
  int32_t pair[NT];
  float wt[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    arow[t] = r_first + t;
    pair[t] = a.row_pair[r_first + t];
    wt[t] = a.topk_w ? a.topk_w[pair[t]] : 1.0f;
  }
  const uint8_t* wc = a.w2_codes + int64_t(e) * H * (I / 2);
  const uint8_t* wsf = a.w2_sf + int64_t(e) * H * (I / 16);
#pragma unroll
  for (int G = 0; G < GROUPS; ++G) {
    float tot[8][NT];
    warp_dot8<L, NT>(wc, wsf, item_row0 + G * 8 * RP, H, a.h_codes, a.h_sf, arow, I, c0, c1, tot);
    if (lane % L == 0) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int64_t n = item_row0 + G * 8 * RP + q * RP + lane / L;
        if (n < H) {
#pragma unroll
          for (int t = 0; t < NT; ++t) slots[int64_t(pair[t]) * H + n] = tot[q][t] * sc * wt[t];
        }
      }
    }
  }
}

template <int L>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kMinCtas) gemv_down_kernel(GemvDownArgs a) {
  const int warp = threadIdx.x >> 5;
  const int64_t H = a.H, I = a.I;
  const int64_t row_groups = (H + 31) / 32;
  const int64_t per_expert = row_groups * a.ksplit;
  const int64_t n_items = int64_t(a.active[0]) * per_expert;
  const int64_t nchunks = I / 32;
  const int64_t cps = ((nchunks + a.ksplit - 1) / a.ksplit + L - 1) / L * L;
  for (int64_t item = int64_t(blockIdx.x) * kWarpsPerCta + warp; item < n_items;
       item += int64_t(gridDim.x) * kWarpsPerCta) {
    const int e = a.active[1 + item / per_expert];
    const int64_t rest = item % per_expert;
    const int64_t split = rest / row_groups;
    const int64_t row0 = (rest % row_groups) * 32;
    const int64_t c0 = split * cps;
    const int64_t c1 = c0 + cps < nchunks ? c0 + cps : nchunks;
    float* slots = a.slots + split * a.slot_stride;
    const int64_t r0 = a.offsets[e], n_e = a.offsets[e + 1] - r0;
    const float sc = a.h_scale[e] * a.w2_scale[e];
    int64_t g = 0;
    for (; g + 2 <= n_e; g += 2) down_group<L, 2>(a, e, row0, r0 + g, c0, c1, sc, slots);
    if (g < n_e) down_group<L, 1>(a, e, row0, r0 + g, c0, c1, sc, slots);
  }
}

// --------------------------------------------------------------- combine ----
// out[t][n] = bf16( sum_j sum_s slots[s][t*k + j][n] (+ shared[t][n]) ), j and s ascending;
// pairs whose row is -1 (skipped ids) contribute nothing.  shared (nullable): the shared
// expert's fp32 output rows, added last.
__device__ __forceinline__ void add_shared(float (&acc)[8], const float* shared, int64_t off) {
  if (!shared) return;
  const float4 a = *reinterpret_cast<const float4*>(shared + off);
  const float4 b = *reinterpret_cast<const float4*>(shared + off + 4);
  acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
  acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
}

__global__ void combine_kernel(const float* __restrict__ slots, int64_t slot_stride, int ksplit,
                               const int32_t* __restrict__ pair_to_row, int T, int H, int k,
                               const float* __restrict__ shared, __nv_bfloat16* __restrict__ out) {
  (void)pair_to_row;  // every pair has a row: slots are addressed by pair directly
  griddep_wait();     // the slot rows come from the down GEMM launched just before
  const int64_t per_row = H / 8;
  const int64_t total = int64_t(T) * per_row;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_row, n = (i - t * per_row) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j0 = 0; j0 < k; j0 += 8) {
      for (int s = 0; s < ksplit; ++s) {
        // up to eight slots' rows in flight at once; summed in slot order
        float4 a[8], b[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (j0 + u < k) {
            const float4* src = reinterpret_cast<const float4*>(slots + s * slot_stride + (t * k + j0 + u) * H + n);
            a[u] = src[0];
            b[u] = src[1];
          }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (j0 + u < k) {
            acc[0] += a[u].x; acc[1] += a[u].y; acc[2] += a[u].z; acc[3] += a[u].w;
            acc[4] += b[u].x; acc[5] += b[u].y; acc[6] += b[u].z; acc[7] += b[u].w;
          }
      }
    }
    add_shared(acc, shared, t * H + n);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
      ow[q] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(out + t * H + n) = o;
  }
}


template <typename K>
int grid_for(K kernel, int64_t warp_items) {
  static std::atomic<int> occ_cache[64];  // zero-initialised; 0 = not queried yet
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = (dev >= 0 && dev < 64) ? occ_cache[dev].load(std::memory_order_relaxed) : 0;
  if (occ == 0) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kWarpsPerCta * 32, 0);
    if (occ < 1) occ = 1;
    if (dev >= 0 && dev < 64) occ_cache[dev].store(occ, std::memory_order_relaxed);  // same value on every thread
  }
  const int64_t full = int64_t(num_sms()) * occ;
  const int64_t need = (warp_items + kWarpsPerCta - 1) / kWarpsPerCta;
  return static_cast<int>(need < full ? (need > 0 ? need : 1) : full);
}

}  // namespace

int gemv_lanes_per_row(int64_t K) {
  const int64_t chunks = K / 32;
  return chunks >= 32 ? 32 : (chunks >= 16 ? 16 : 8);
}

nvfp4moe_status launch_gemv_gateup(const GemvGateUpArgs& a, int64_t max_active, cudaStream_t s) {
  const int L = gemv_lanes_per_row(a.H);
  const int64_t items = max_active * (2 * int64_t(a.I) / 32);
  if (L == 32)
    gemv_gateup_kernel<32><<<grid_for(gemv_gateup_kernel<32>, items), kWarpsPerCta * 32, 0, s>>>(a);
  else if (L == 16)
    gemv_gateup_kernel<16><<<grid_for(gemv_gateup_kernel<16>, items), kWarpsPerCta * 32, 0, s>>>(a);
  else
    gemv_gateup_kernel<8><<<grid_for(gemv_gateup_kernel<8>, items), kWarpsPerCta * 32, 0, s>>>(a);
  return check_launch("gemv gate/up");
}

int gemv_down_ksplit(int64_t max_active, int64_t H, int64_t I) {
  const int L = gemv_lanes_per_row(I);
  const int64_t items = max_active * ((H + 31) / 32);
  if (items <= 0) return 1;  // an empty batch
  const int64_t want = int64_t(num_sms()) * 16;
  int64_t ks = (want + items - 1) / items;
  const int64_t max_ks = (I / 32) / L;
  if (ks > max_ks) ks = max_ks;
  if (ks < 1) ks = 1;
  if (ks > 32) ks = 32;
  return static_cast<int>(ks);
}

nvfp4moe_status launch_gemv_down(const GemvDownArgs& a, int64_t max_active, cudaStream_t s) {
  const int L = gemv_lanes_per_row(a.I);
  const int64_t items = max_active * ((int64_t(a.H) + 31) / 32) * a.ksplit;
  if (L == 32)
    gemv_down_kernel<32><<<grid_for(gemv_down_kernel<32>, items), kWarpsPerCta * 32, 0, s>>>(a);
  else if (L == 16)
    gemv_down_kernel<16><<<grid_for(gemv_down_kernel<16>, items), kWarpsPerCta * 32, 0, s>>>(a);
  else
    gemv_down_kernel<8><<<grid_for(gemv_down_kernel<8>, items), kWarpsPerCta * 32, 0, s>>>(a);
  return check_launch("gemv down");
}

nvfp4moe_status launch_combine(const float* slots, int64_t slot_stride, int ksplit,
                               const int32_t* pair_to_row, int T, int H, int k, void* out,
                               cudaStream_t s, const float* shared) {
  const int64_t total = int64_t(T) * (H / 8);
  if (total == 0) return NVFP4MOE_OK;
  int64_t blocks = (total + 255) / 256;
  if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
  const cudaError_t e = launch_dependent(combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, slots,
                                         slot_stride, ksplit, pair_to_row, T, H, k, shared,
                                         static_cast<__nv_bfloat16*>(out));
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "combine: %s", cudaGetErrorString(e));
  return check_launch("combine");
}

__global__ void combine_rows_kernel(const float* __restrict__ slots, const int32_t* __restrict__ pair_to_row,
                                    const float* __restrict__ topk_w, int T, int H, int k,
                                    const float* __restrict__ shared, __nv_bfloat16* __restrict__ out) {
  griddep_wait();  // the slot rows come from the down GEMM launched just before
  const int64_t per_row = H / 8;
  const int64_t total = int64_t(T) * per_row;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_row, n = (i - t * per_row) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j0 = 0; j0 < k; j0 += 8) {
      int32_t row[8];
      float wj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        row[u] = j0 + u < k ? __ldg(pair_to_row + t * k + j0 + u) : 0;
        wj[u] = j0 + u < k ? __ldg(topk_w + t * k + j0 + u) : 0.0f;
      }
      float4 a[8], b[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u < k) {
          const float4* src = reinterpret_cast<const float4*>(slots + int64_t(row[u]) * H + n);
          a[u] = src[0];
          b[u] = src[1];
        }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u < k) {  // in slot order
          acc[0] += wj[u] * a[u].x; acc[1] += wj[u] * a[u].y; acc[2] += wj[u] * a[u].z; acc[3] += wj[u] * a[u].w;
          acc[4] += wj[u] * b[u].x; acc[5] += wj[u] * b[u].y; acc[6] += wj[u] * b[u].z; acc[7] += wj[u] * b[u].w;
        }
    }
    add_shared(acc, shared, t * H + n);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
      ow[q] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(out + t * H + n) = o;
  }
}

nvfp4moe_status launch_combine_rows(const float* slots, const int32_t* pair_to_row, const float* topk_w, int T, int H,
                                    int k, void* out, cudaStream_t s, const float* shared) {
  const int64_t total = int64_t(T) * (H / 8);
  if (total == 0) return NVFP4MOE_OK;
  int64_t blocks = (total + 255) / 256;
  if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
  const cudaError_t e = launch_dependent(combine_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, slots,
                                         pair_to_row, topk_w, T, H, k, shared, static_cast<__nv_bfloat16*>(out));
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "combine (rows): %s", cudaGetErrorString(e));
  return check_launch("combine (rows)");
}

__global__ void accum_to_bf16_kernel(const float* __restrict__ acc, int64_t n, const float* __restrict__ shared,
                                     __nv_bfloat16* __restrict__ out) {
  griddep_wait();  // the accumulator is complete when the down GEMM is
  for (int64_t i = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) * 8; i < n; i += int64_t(gridDim.x) * blockDim.x * 8) {
    float4 a = *reinterpret_cast<const float4*>(acc + i);
    float4 b = *reinterpret_cast<const float4*>(acc + i + 4);
    if (shared) {  // the shared expert's rows, added last
      const float4 sa = *reinterpret_cast<const float4*>(shared + i), sb = *reinterpret_cast<const float4*>(shared + i + 4);
      a = make_float4(a.x + sa.x, a.y + sa.y, a.z + sa.z, a.w + sa.w);
      b = make_float4(b.x + sb.x, b.y + sb.y, b.z + sb.z, b.w + sb.w);
    }
    const __nv_bfloat162 q0 = __floats2bfloat162_rn(a.x, a.y), q1 = __floats2bfloat162_rn(a.z, a.w);
    const __nv_bfloat162 q2 = __floats2bfloat162_rn(b.x, b.y), q3 = __floats2bfloat162_rn(b.z, b.w);
    *reinterpret_cast<uint4*>(out + i) =
        make_uint4(*reinterpret_cast<const uint32_t*>(&q0), *reinterpret_cast<const uint32_t*>(&q1),
                   *reinterpret_cast<const uint32_t*>(&q2), *reinterpret_cast<const uint32_t*>(&q3));
  }
}

nvfp4moe_status launch_accum_to_bf16(const float* acc, int64_t n, void* out, cudaStream_t s, const float* shared) {
  if (n == 0) return NVFP4MOE_OK;
  int64_t blocks = (n / 8 + 255) / 256;
  if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
  const cudaError_t e = launch_dependent(accum_to_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, acc, n,
                                         shared, static_cast<__nv_bfloat16*>(out));
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "accumulator to bf16: %s", cudaGetErrorString(e));
  return check_launch("accumulator to bf16");
}

}  // namespace nvfp4moe
