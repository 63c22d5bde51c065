// Dense bf16 GEMMs of the shared expert on the tensor cores (tcgen05.mma kind::f16), for
// batches too large for the streamed CUDA-core kernel.
//
// The shared expert (the SSD-Stream card keeps the shared experts in BF16) is one dense
// SwiGLU MLP applied to every token: gate/up D[2I_s][T] = W13 . x^T, then down
// D[H][T] = W2 . h^T.  As in the routed kernels the weights are the MMA's M operand (128 rows
// per tile) and the tokens its N operand (chunks of 128 tokens; rows past T are zeros from
// the TMA fill).  Both operands are K-major bf16 tiles of 128 rows x 128 bytes (64 elements)
// with the 128-byte swizzle, six stages in shared memory; fp32 accumulators in TMEM (two
// of 128 columns).
//   warp 0      TMA producer (weight tile and token tile of each stage, one barrier);
//   warp 1      TMEM owner and MMA issuer: four K = 16 MMAs per stage;
//   warps 2..5  epilogue, one 32-row TMEM lane quarter each: gate/up applies SwiGLU (gate
//               and up rows are lanes i and 16+i of the same warp by the W13 interleave) and
//               stores h in bf16 [T][I_s]; down stores its fp32 rows [T][H] for the combine.
// Every wait is bounded (status bit on timeout; copies in flight land before the CTA exits).
#include "ffn_gemv.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int DM = 128;           // weight rows per tile
constexpr int DBN = 128;          // tokens per chunk
constexpr int DSTAGES = 6;
constexpr int DTHREADS = 192;
constexpr int D_A_BYTES = DM * 128;
constexpr int D_B_BYTES = DBN * 128;
constexpr uint32_t kDTimeout = 1u << 3;

__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// kind::f16 instruction descriptor: fp32 accumulator (bits [4,6) = 1), bf16 A and B (bits
// [7,10) and [10,13) = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

struct DenseParams {
  int K, NW, T;       // reduction, weight rows, tokens
  uint16_t* h_out;    // EPI 0: bf16 [T][NW / 2]
  float* y_out;       // EPI 1: fp32 [T][NW]
  uint32_t* status;
};

template <int EPI>
__global__ void __launch_bounds__(DTHREADS, 1)
dense_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, DenseParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + DSTAGES * D_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + DSTAGES * D_B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = full + DSTAGES;
  uint64_t* acc_full = empty + DSTAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < DSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  griddep_wait();  // the tokens (x, or h from the gate/up launch) come from earlier kernels
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_mt = p.NW / DM, n_ch = (p.T + DBN - 1) / DBN, kt_n = p.K / 64;
  const int n_items = n_mt * n_ch;
  auto abort_now = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kDTimeout);
  };

  if (warp == 0) {
    if (elect_one()) {
      uint32_t it = 0;
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        const int mt = item / n_ch, ch = item - mt * n_ch;
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = it % DSTAGES;
          if (!mbar_wait(&empty[s], ((it / DSTAGES) & 1) ^ 1)) {
            abort_now();
            break;
          }
          mbar_arrive_expect_tx(&full[s], D_A_BYTES + D_B_BYTES);
          tma_load_2d(sA + s * D_A_BYTES, &tmA, kt * 128, mt * DM, &full[s]);
          tma_load_2d(sB + s * D_B_BYTES, &tmB, kt * 128, ch * DBN, &full[s]);
        }
      }
      if (*abort_flag)
        for (uint32_t back = 0; back < DSTAGES && back < it; ++back) {
          const uint32_t jj = it - 1 - back;
          mbar_wait(&full[jj % DSTAGES], (jj / DSTAGES) & 1, 1u << 16);
        }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16(DM, DBN);
      uint32_t it = 0, li = 0;
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x, ++li) {
        const uint32_t ab = li & 1;
        if (!mbar_wait(&acc_empty[ab], ((li >> 1) & 1) ^ 1)) {
          abort_now();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = it % DSTAGES;
          if (!mbar_wait(&full[s], (it / DSTAGES) & 1)) {
            abort_now();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_d = desc_kmajor_sw128(sA + s * D_A_BYTES);
          const uint64_t b_d = desc_kmajor_sw128(sB + s * D_B_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j)  // K = 16 per MMA: 32 bytes = 2 descriptor units
            tc_mma_bf16(tmem + ab * DBN, a_d + 2 * j, b_d + 2 * j, idesc, (kt | j) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, 1u << 20);
    }
  } else {
    const int q = warp & 3;  // the TMEM lane quarter this warp may read
    const uint32_t trow = tmem + (uint32_t(q * 32) << 16);
    uint32_t li = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++li) {
      const int mt = item / n_ch, ch = item - mt * n_ch;
      const uint32_t ab = li & 1;
      if (*abort_flag || !mbar_wait(&acc_full[ab], (li >> 1) & 1)) {
        abort_now();
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < DBN / 32; ++cc) {
        const int tok0 = ch * DBN + cc * 32;
        if (tok0 >= p.T) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(trow + ab * DBN + cc * 32, r);
        tmem_ld_wait();
        if (EPI == 0) {
          // lanes 0..15: gate rows 32q+l of h block mt*4+q; lanes 16..31: the matching up rows
          const int I = p.NW / 2;
          const int col = (mt * 4 + q) * 16 + (lane & 15);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float mine = __uint_as_float(r[j]);
            const float up = __shfl_down_sync(0xffffffffu, mine, 16);
            if (lane < 16 && tok0 + j < p.T) {
              const float h = mine / (1.0f + expf(-mine)) * up;
              const __nv_bfloat16 hb = __float2bfloat16_rn(h);
              p.h_out[int64_t(tok0 + j) * I + col] = *reinterpret_cast<const uint16_t*>(&hb);
            }
          }
        } else {
          const int n = mt * DM + q * 32 + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (tok0 + j < p.T) p.y_out[int64_t(tok0 + j) * p.NW + n] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

}  // namespace

// epi 0: h_out[T][NW/2] = bf16(silu(W13 . x) * (W13 . x)) (interleaved rows), epi 1:
// y_out[T][NW] = W2 . h.  weights bf16 [NW][K], act bf16 [T][K].
nvfp4moe_status launch_dense_bf16(int epi, const uint16_t* weights, const uint16_t* act, int K, int NW, int T,
                                  uint16_t* h_out, float* y_out, cudaStream_t s) {
  uint32_t* status = device_status_ptr();
  if (!status) return fail(NVFP4MOE_CUDA_ERROR, "device status word unavailable");
  if (T <= 0) return NVFP4MOE_OK;
  if (K % 64 != 0 || NW % DM != 0)
    return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "dense bf16 GEMM: K=%d, rows=%d", K, NW);
  // bf16 rows are 2K bytes: the FP4 code-map helper describes them as K' = 4K elements
  CUtensorMap a_map, b_map;
  nvfp4moe_status st = make_code_map(&a_map, weights, NW, int64_t(4) * K, DM);
  if (st == NVFP4MOE_OK) st = make_code_map(&b_map, act, T, int64_t(4) * K, DBN);
  if (st != NVFP4MOE_OK) return st;
  DenseParams p{};
  p.K = K;
  p.NW = NW;
  p.T = T;
  p.h_out = h_out;
  p.y_out = y_out;
  p.status = status;
  const size_t smem = 1024 + size_t(DSTAGES) * (D_A_BYTES + D_B_BYTES) + (2 * DSTAGES + 5) * 8 + 16;
  const int64_t items = int64_t(NW / DM) * ((T + DBN - 1) / DBN);
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e == cudaSuccess) e = launch_dependent(kern, dim3(grid), dim3(DTHREADS), smem, s, a_map, b_map, p);
    return e;
  };
  const cudaError_t e = epi == 0 ? go(dense_bf16_kernel<0>) : go(dense_bf16_kernel<1>);
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "dense bf16 GEMM: %s", cudaGetErrorString(e));
  return check_launch("dense bf16 GEMM");
}

}  // namespace nvfp4moe
