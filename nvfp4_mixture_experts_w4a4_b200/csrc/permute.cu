// moe_permute: expert histogram + prefix scan + stable placement of (token, slot) pairs
// into per-expert row groups, in one CTA.
//
// The tokens are split into W contiguous chunks, one per warp.  A warp takes 32/k whole
// tokens per step (lane = token_in_step * k + slot), so lanes in ascending order are pairs in
// ascending token order.  Pass 1: each warp counts its chunk's pairs per expert into
// hist[w][e] (lanes naming the same expert in one step are grouped with __match_any_sync and
// the lowest of them adds the group size).  Scan: hist[w][e] becomes the number of pairs of
// expert e in chunks before w, and counts / offsets / padded offsets come from a scan over
// experts.  Pass 2: the warps walk their chunks again; a pair's row is padded_offsets[e] +
// hist[w][e] + (number of lower lanes of this step with the same expert).  The result is
// the unique stable order (experts ascending, tokens ascending inside an expert) without
// global atomics, so it is deterministic.
#include "common.cuh"

namespace nvfp4moe {
namespace {

constexpr int kThreads = 1024;

// Lane (token_in_step * k + slot) owns one pair of the step's tokens [t0, t0 + per_step).
// Returns the pair index (or -1 for idle lanes) and the expert in *e (-1 if the id is out of
// range or repeats an id of a lower slot of the same token; both flag the status word).
__device__ __forceinline__ int64_t step_pair(const int32_t* ids, int t0, int t_end, int k, int E, uint32_t* status,
                                             int* e_out) {
  const int lane = threadIdx.x & 31;
  const int per_step = 32 / k;
  const int tl = lane / k, j = lane - tl * k;
  const int t = t0 + tl;
  const bool live = tl < per_step && t < t_end;
  const int64_t p = live ? int64_t(t) * k + j : -1;
  int e = live ? ids[p] : -1;
  const bool bad = live && (e < 0 || e >= E);
  if (bad) {
    atomicOr(status, uint32_t(NVFP4MOE_DEV_BAD_EXPERT_ID));
    e = -1;
  }
  // a duplicate is a lower slot of the same token with the same expert
  const unsigned same = __match_any_sync(0xffffffffu, live ? e : -2 - lane);
  const unsigned mine = k >= 32 ? 0xffffffffu : ((1u << k) - 1u) << (tl * k);  // lanes of this token
  if (live && e >= 0 && (same & mine & ((1u << lane) - 1u)) != 0u) {
    atomicOr(status, uint32_t(NVFP4MOE_DEV_DUPLICATE_ID));
    e = -1;
  }
  *e_out = e;
  return p;
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

template <int W>
__global__ void __launch_bounds__(kThreads)
permute_kernel(const int32_t* __restrict__ ids, int T, int E, int k, int m_tile, int64_t rows_cap,
               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
               int32_t* __restrict__ padded_offsets, int32_t* __restrict__ pair_to_row,
               int32_t* __restrict__ row_token, int32_t* __restrict__ row_pair,
               int32_t* __restrict__ tile_expert, int32_t* __restrict__ active,
               float* __restrict__ zero_f32, uint32_t* __restrict__ status) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;                    // [W][E]
  int32_t* cnt = hist + W * E;             // [E]
  int32_t* padc = cnt + E;                 // [E]
  int32_t* off = padc + E;                 // [E+1]
  int32_t* poff = off + E + 1;             // [E+1]
  int32_t* flag = poff + E + 1;            // [E]
  int32_t* aoff = flag + E;                // [E+1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool worker = warp < W;

  for (int i = tid; i < W * E; i += kThreads) hist[i] = 0;
  if (zero_f32)
    for (int i = tid; i < E; i += kThreads) zero_f32[i] = 0.0f;
  __syncthreads();

  const int chunk = (T + W - 1) / W;
  const int t0 = warp * chunk;
  const int t1 = min(T, t0 + chunk);
  const int per_step = 32 / k;
  int32_t* my = hist + warp * E;
  if (worker) {
    for (int t = t0; t < t1; t += per_step) {
      int e;
      step_pair(ids, t, t1, k, E, status, &e);
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && (grp & ((1u << lane) - 1u)) == 0u) my[e] += __popc(grp);
      __syncwarp();
    }
  }
  __syncthreads();

  for (int e = tid; e < E; e += kThreads) {
    int32_t run = 0;
    for (int w = 0; w < W; ++w) {
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
  if (worker) {
    for (int t = t0; t < t1; t += per_step) {
      int e;
      const int64_t p = step_pair(ids, t, t1, k, E, status, &e);
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(grp & ((1u << lane) - 1u));
      if (p >= 0) {
        int32_t row = -1;
        if (e >= 0 && fits) {
          row = poff[e] + my[e] + rank;
          row_token[row] = static_cast<int32_t>(p / k);
          row_pair[row] = static_cast<int32_t>(p);
        }
        pair_to_row[p] = row;
      }
      __syncwarp();
      if (e >= 0 && rank == 0) my[e] += __popc(grp);
      __syncwarp();
    }
  }
  __syncthreads();

  for (int e = tid; e < E; e += kThreads) {
    counts[e] = cnt[e];
    offsets[e] = off[e];
    padded_offsets[e] = poff[e];
    if (flag[e]) active[1 + aoff[e]] = e;
  }
  if (fits) {
    // padding rows and the tile -> expert map, spread over all threads
    for (int e = warp; e < E; e += kThreads / 32) {
      for (int r = poff[e] + cnt[e] + lane; r < poff[e + 1]; r += 32) {
        row_token[r] = -1;
        row_pair[r] = -1;
      }
      for (int tl = poff[e] / m_tile + lane; tl < poff[e + 1] / m_tile; tl += 32) tile_expert[tl] = e;
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
  NVFP4_REQUIRE(m_tile == 1 || m_tile == 32 || m_tile == 64 || m_tile == 128, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: m_tile must be 1, 32, 64 or 128", fn);
  NVFP4_REQUIRE(int64_t(T) * k <= (int64_t(1) << 24), NVFP4MOE_UNSUPPORTED_SHAPE, "%s: T*k > 2^24", fn);
  NVFP4_REQUIRE(rows_cap >= moe_permute_rows_capacity(T, E, k, m_tile), NVFP4MOE_INVALID_ARG,
                "%s: rows_cap %lld < capacity %lld", fn, (long long)rows_cap,
                (long long)moe_permute_rows_capacity(T, E, k, m_tile));
  NVFP4_REQUIRE(counts && offsets && padded_offsets && active, NVFP4MOE_INVALID_ARG, "%s: NULL output", fn);
  NVFP4_REQUIRE(T == 0 || (ids && pair_to_row && row_token && row_pair && tile_expert),
                NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  uint32_t* status = device_status_ptr();
  NVFP4_REQUIRE(status != nullptr, NVFP4MOE_CUDA_ERROR, "%s: device status word unavailable", fn);
  const int W = E <= 512 ? 32 : 16;  // warps with a private histogram (smem: W*E ints)
  const size_t smem = sizeof(int32_t) * (size_t(W) * E + 6 * size_t(E) + 3);
  cudaError_t attr = set_smem_limit_once<permute_kernel<32>>(100 * 1024);
  if (attr == cudaSuccess) attr = set_smem_limit_once<permute_kernel<16>>(100 * 1024);
  NVFP4_REQUIRE(attr == cudaSuccess, NVFP4MOE_CUDA_ERROR, "%s: shared-memory attribute: %s", fn,
                cudaGetErrorString(attr));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (W == 32)
    permute_kernel<32><<<1, kThreads, smem, s>>>(ids, T, E, k, m_tile, rows_cap, counts, offsets, padded_offsets,
                                                  pair_to_row, row_token, row_pair, tile_expert, active, zero_f32,
                                                  status);
  else
    permute_kernel<16><<<1, kThreads, smem, s>>>(ids, T, E, k, m_tile, rows_cap, counts, offsets, padded_offsets,
                                                  pair_to_row, row_token, row_pair, tile_expert, active, zero_f32,
                                                  status);
  return check_launch(fn);
}

}  // extern "C"
