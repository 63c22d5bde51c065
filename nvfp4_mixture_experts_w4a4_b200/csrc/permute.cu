// moe_permute: expert histogram + prefix scan + stable placement of (token, slot) pairs
// into per-expert row groups, in one CTA.
//
// The tokens are split into kWarps contiguous chunks.  Pass 1: warp w counts its chunk's
// pairs per expert into hist[w][e] (a token never names an expert twice, so the lanes of
// one token touch distinct counters).  Scan: hist[w][e] becomes the number of pairs of
// expert e in chunks before w, and counts / offsets / padded offsets come from a scan over
// experts.  Pass 2: warp w walks its chunk again in token order and hands out rows
// padded_offsets[e] + hist[w][e]++.  The result is the unique stable order (experts
// ascending, tokens ascending inside an expert) with no atomics, so it is deterministic.
#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;

// Lane j < k owns pair (t, j).  Returns the expert, or -1 if the id is out of range or
// repeats an id of a lower slot of the same token (both flag the status word).
__device__ __forceinline__ int valid_expert(const int32_t* ids, int64_t p, int lane, int k, int E,
                                            uint32_t* status) {
  const unsigned active = (k >= 32) ? 0xffffffffu : ((1u << k) - 1u);
  int e = (lane < k) ? ids[p] : -1;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  if (lane >= k) return -1;
  if (e < 0 || e >= E) {
    atomicOr(status, uint32_t(NVFP4MOE_DEV_BAD_EXPERT_ID));
    return -1;
  }
  if ((same & active & ((1u << lane) - 1u)) != 0u) {
    atomicOr(status, uint32_t(NVFP4MOE_DEV_DUPLICATE_ID));
    return -1;
  }
  return e;
}

// Exclusive scan of in[0..n) into out[0..n] by warp 0 (out[n] = total).
__device__ void warp_exclusive_scan(const int32_t* in, int32_t* out, int n) {
  const int lane = threadIdx.x & 31;
  int32_t carry = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int32_t v = i < n ? in[i] : 0;
    int32_t s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (i < n) out[i] = carry + s - v;
    carry += __shfl_sync(0xffffffffu, s, 31);
  }
  if (lane == 0) out[n] = carry;
}

__global__ void __launch_bounds__(kThreads)
permute_kernel(const int32_t* __restrict__ ids, int T, int E, int k, int m_tile, int64_t rows_cap,
               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
               int32_t* __restrict__ padded_offsets, int32_t* __restrict__ pair_to_row,
               int32_t* __restrict__ row_token, int32_t* __restrict__ row_pair,
               int32_t* __restrict__ tile_expert, int32_t* __restrict__ active,
               float* __restrict__ zero_f32, uint32_t* __restrict__ status) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;                    // [kWarps][E]
  int32_t* cnt = hist + kWarps * E;        // [E]
  int32_t* padc = cnt + E;                 // [E]
  int32_t* off = padc + E;                 // [E+1]
  int32_t* poff = off + E + 1;             // [E+1]
  int32_t* flag = poff + E + 1;            // [E]
  int32_t* aoff = flag + E;                // [E+1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < kWarps * E; i += kThreads) hist[i] = 0;
  if (zero_f32)
    for (int i = tid; i < E; i += kThreads) zero_f32[i] = 0.0f;
  __syncthreads();

  const int chunk = (T + kWarps - 1) / kWarps;
  const int t0 = warp * chunk;
  const int t1 = min(T, t0 + chunk);
  int32_t* my = hist + warp * E;
  for (int t = t0; t < t1; ++t) {
    const int e = valid_expert(ids, int64_t(t) * k + lane, lane, k, E, status);
    if (e >= 0) my[e] += 1;
    __syncwarp();
  }
  __syncthreads();

  for (int e = tid; e < E; e += kThreads) {
    int32_t run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int32_t c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    cnt[e] = run;
    padc[e] = (run + m_tile - 1) / m_tile * m_tile;
    flag[e] = run > 0 ? 1 : 0;
  }
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(cnt, off, E);
  if (warp == 1) warp_exclusive_scan(padc, poff, E);
  if (warp == 2) warp_exclusive_scan(flag, aoff, E);
  __syncthreads();

  const bool fits = int64_t(poff[E]) <= rows_cap;
  if (!fits && tid == 0) atomicOr(status, uint32_t(NVFP4MOE_DEV_ROW_OVERFLOW));
  for (int t = t0; t < t1; ++t) {
    const int64_t p = int64_t(t) * k + lane;
    const int e = valid_expert(ids, p, lane, k, E, status);
    if (lane < k) {
      int32_t row = -1;
      if (e >= 0 && fits) {
        row = poff[e] + my[e];
        my[e] += 1;
        row_token[row] = t;
        row_pair[row] = static_cast<int32_t>(p);
      }
      pair_to_row[p] = row;
    }
    __syncwarp();
  }

  for (int e = tid; e < E; e += kThreads) {
    counts[e] = cnt[e];
    offsets[e] = off[e];
    padded_offsets[e] = poff[e];
    if (flag[e]) active[1 + aoff[e]] = e;
    if (fits) {
      for (int r = poff[e] + cnt[e]; r < poff[e + 1]; ++r) {
        row_token[r] = -1;
        row_pair[r] = -1;
      }
      for (int tl = poff[e] / m_tile; tl < poff[e + 1] / m_tile; ++tl) tile_expert[tl] = e;
    }
  }
  if (tid == 0) {
    offsets[E] = off[E];
    padded_offsets[E] = fits ? poff[E] : 0;
    active[0] = aoff[E];
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

int64_t moe_permute_rows_capacity(int32_t T, int32_t E, int32_t k, int32_t m_tile) {
  if (T < 0 || E < 1 || k < 1 || m_tile < 1) return 0;
  const int64_t P = int64_t(T) * k;
  const int64_t groups = P < E ? P : E;
  return P + groups * (m_tile - 1);
}

nvfp4moe_status moe_permute(const int32_t* ids, int32_t T, int32_t E, int32_t k, int32_t m_tile,
                            int64_t rows_cap, int32_t* counts, int32_t* offsets,
                            int32_t* padded_offsets, int32_t* pair_to_row, int32_t* row_token,
                            int32_t* row_pair, int32_t* tile_expert, int32_t* active,
                            float* zero_f32, nvfp4moe_stream_t stream) {
  const char* fn = "moe_permute";
  NVFP4_REQUIRE(T >= 0, NVFP4MOE_INVALID_ARG, "%s: T < 0", fn);
  NVFP4_REQUIRE(E >= 1 && E <= 1024, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: E=%d outside [1, 1024]", fn, E);
  NVFP4_REQUIRE(k >= 1 && k <= 32 && k <= E, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: bad k=%d", fn, k);
  NVFP4_REQUIRE(m_tile == 1 || m_tile == 128, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: m_tile must be 1 or 128", fn);
  NVFP4_REQUIRE(int64_t(T) * k <= (int64_t(1) << 24), NVFP4MOE_UNSUPPORTED_SHAPE, "%s: T*k > 2^24", fn);
  NVFP4_REQUIRE(rows_cap >= moe_permute_rows_capacity(T, E, k, m_tile), NVFP4MOE_INVALID_ARG,
                "%s: rows_cap %lld < capacity %lld", fn, (long long)rows_cap,
                (long long)moe_permute_rows_capacity(T, E, k, m_tile));
  NVFP4_REQUIRE(counts && offsets && padded_offsets && active, NVFP4MOE_INVALID_ARG, "%s: NULL output", fn);
  NVFP4_REQUIRE(T == 0 || (ids && pair_to_row && row_token && row_pair && tile_expert),
                NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  uint32_t* status = device_status_ptr();
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_CUDA_ERROR, "%s: device status word unavailable", fn);
  const size_t smem = sizeof(int32_t) * (size_t(kWarps) * E + 6 * size_t(E) + 3);
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024);
    configured[dev] = 1;
  }
  permute_kernel<<<1, kThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      ids, T, E, k, m_tile, rows_cap, counts, offsets, padded_offsets, pair_to_row, row_token,
      row_pair, tile_expert, active, zero_f32, status);
  return check_launch(fn);
}

}  // extern "C"
