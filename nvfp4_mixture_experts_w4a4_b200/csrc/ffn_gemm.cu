// nvfp4_gemm on tcgen05 block-scaled MMA (.kind::mxf4nvf4, E2M1 operands, UE4M3 scales
// per 16 elements, fp32 accumulation in TMEM): D[M][N] = A . B^T * a_scale * b_scale.
//
// One persistent CTA per SM walks the output tiles (128 rows of A x BN rows of B) with a
// static stride, row-tile-major, so the CTAs of one wave share an A tile.  Warp roles:
//   warp 0      one elected thread issues TMA loads of the A and B code tiles (128-byte
//               swizzle, 256 K-elements = 128 bytes per row per stage) and bulk copies of
//               their 512-byte scale atoms into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns, and one elected thread copies each stage's
//               scales to TMEM (tcgen05.cp) and issues four K=64 MMAs per stage into the
//               fp32 accumulator (TMEM columns [0, BN)), then commits;
//   warps 2..5  the epilogue: each warp reads its 32 TMEM lanes (= 32 rows) in
//               32-column slices, scales them and stores bf16 or fp32 D.
// Every wait is bounded: on a timeout the CTA raises a status bit, drains what it issued
// and returns instead of spinning.
#include "ffn_gemm.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 256;            // K elements per stage
constexpr int KB = BK / 2;         // bytes of codes per row per stage (= swizzle span)
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDevTimeout = 1u << 3;


struct GemmParams {
  int K, N, M;
  int num_m;
  const uint8_t* a_sf;
  const uint8_t* b_sf;
  const float* a_scale;
  const float* b_scale;
  void* D;
  int d_f32;
  uint32_t* status;
};

template <int BN>
struct Smem {
  static constexpr int A = BM * KB;
  static constexpr int B = BN * KB;
  static constexpr int SFA = BM * BK / 16;
  static constexpr int SFB = BN * BK / 16;
  static constexpr int STAGE = A + B + SFA + SFB;
  static constexpr int BARS = 2 * STAGES + 3;
  static constexpr int BYTES = 1024 + STAGES * STAGE + BARS * 8 + 16;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using S = Smem<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * S::A;
  uint8_t* sSFA = sB + STAGES * S::B;
  uint8_t* sSFB = sSFA + STAGES * S::SFA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + STAGES * S::SFB);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + S::BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4 * 32);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int num_m = p.num_m;
  const int n_tiles = p.N / BN;
  const int total = num_m * n_tiles;
  const int k_tiles = (p.K + BK - 1) / BK;
  const int64_t katoms = p.K / 64;  // 64-element scale atoms along K
  auto abort_now = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kDevTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    if (elect_one()) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
        const int mt = t / n_tiles, nt = t % n_tiles;
        const uint8_t* bsf = p.b_sf;
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1)) {
            abort_now();
            break;
          }
          const int nkb = min(4, (p.K - kt * BK) / 64);
          const uint32_t sf_bytes = nkb * 512;
          mbar_arrive_expect_tx(&full[s], S::A + S::B + sf_bytes * (1 + BN / 128));
          tma_load_2d(sA + s * S::A, &tmA, kt * KB, mt * BM, &full[s]);
          tma_load_2d(sB + s * S::B, &tmB, kt * KB, nt * BN, &full[s]);
          bulk_load(sSFA + s * S::SFA, p.a_sf + (int64_t(mt) * katoms + kt * 4) * 512, sf_bytes, &full[s]);
#pragma unroll
          for (int h = 0; h < BN / 128; ++h)
            bulk_load(sSFB + s * S::SFB + h * 2048, bsf + (int64_t(nt * (BN / 128) + h) * katoms + kt * 4) * 512,
                      sf_bytes, &full[s]);
        }
      }
      if (*abort_flag) {
        // let the loads already issued land before the CTA's shared memory goes away
        for (uint32_t back = 0; back < STAGES && back < it; ++back) {
          const uint32_t j = it - 1 - back;
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, 1u << 16);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA ----
    if (elect_one()) {
      const uint32_t idesc = idesc_mxf4nvf4(BM, BN);
      const uint32_t sfa_t = tmem + BN;
      const uint32_t sfb_t = tmem + BN + 16;
      constexpr uint32_t SFB_COLS = 4 * (BN / 128);
      uint32_t it = 0, tc = 0;
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++tc) {
        if (!mbar_wait(acc_empty, (tc & 1) ^ 1)) {
          abort_now();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1)) {
            abort_now();
            ok = false;
            break;
          }
          tc_fence_after();
          const int nkb = min(4, (p.K - kt * BK) / 64);
          for (int j = 0; j < nkb; ++j) {
            tc_cp_sf(sfa_t + 4 * j, desc_sf_atom(sSFA + s * S::SFA + j * 512));
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tc_cp_sf(sfb_t + SFB_COLS * j + 4 * h, desc_sf_atom(sSFB + s * S::SFB + h * 2048 + j * 512));
          }
          const uint64_t a0 = desc_kmajor_sw128(sA + s * S::A);
          const uint64_t b0 = desc_kmajor_sw128(sB + s * S::B);
          for (int j = 0; j < nkb; ++j)
            tc_mma_mxf4nvf4(tmem, a0 + uint64_t(2 * j), b0 + uint64_t(2 * j), idesc, sfa_t + 4 * j,
                            sfb_t + SFB_COLS * j, (kt | j) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      // every MMA issued by this thread has finished before TMEM is released
      tc_commit(drain);
      mbar_wait(drain, 0, 1u << 20);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;  // TMEM sub-partition this warp may read
    const int rt = q * 32 + lane;
    const uint32_t trow = tmem + (uint32_t(q * 32) << 16);
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++tc) {
      if (!mbar_wait(acc_full, tc & 1)) {
        abort_now();
        break;
      }
      tc_fence_after();
      const int mt = t / n_tiles, nt = t % n_tiles;
      const int64_t row = int64_t(mt) * BM + rt;
      {
        const bool valid = row < p.M;
        const float sc = p.a_scale[0] * p.b_scale[0];
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + c * 32, r);
          tmem_ld_wait();
          if (valid) {
            const int64_t col = int64_t(nt) * BN + c * 32;
            if (p.d_f32) {
              float* dst = static_cast<float*>(p.D) + row * p.N + col;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(dst + j) =
                    make_float4(__uint_as_float(r[j]) * sc, __uint_as_float(r[j + 1]) * sc,
                                __uint_as_float(r[j + 2]) * sc, __uint_as_float(r[j + 3]) * sc);
            } else {
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.D) + row * p.N + col;
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[j + 2 * u]) * sc,
                                                                  __uint_as_float(r[j + 2 * u + 1]) * sc);
                  ow[u] = *reinterpret_cast<const uint32_t*>(&b);
                }
                *reinterpret_cast<uint4*>(dst + j) = o;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side ----
template <int BN>
nvfp4moe_status launch(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, int64_t max_tiles,
                       cudaStream_t s) {
  auto kern = gemm_kernel<BN>;
  {
    const cudaError_t e = set_smem_limit_once<gemm_kernel<BN>>(Smem<BN>::BYTES);
    if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "tcgen05 GEMM smem attribute: %s", cudaGetErrorString(e));
  }
  int64_t grid = num_sms();
  if (max_tiles < grid) grid = max_tiles > 0 ? max_tiles : 1;
  kern<<<static_cast<int>(grid), kThreads, Smem<BN>::BYTES, s>>>(a, b, p);
  return check_launch("tcgen05 GEMM");
}

}  // namespace

bool gemm_path_available() { return tensor_map_encoder() != nullptr; }

nvfp4moe_status launch_gemm_plain(const uint8_t* A, const uint8_t* A_sf, const float* a_scale, const uint8_t* B,
                                  const uint8_t* B_sf, const float* b_scale, int64_t M, int64_t N, int64_t K, void* D,
                                  int d_f32, cudaStream_t s) {
  uint32_t* status = device_status_ptr();
  if (!status) return fail(NVFP4MOE_CUDA_ERROR, "device status word unavailable");
  const int BN = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb;
  nvfp4moe_status st = make_code_map(&ta, A, M, K, BM);
  if (st != NVFP4MOE_OK) return st;
  st = make_code_map(&tb, B, N, K, BN);
  if (st != NVFP4MOE_OK) return st;
  GemmParams p{};
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.M = static_cast<int>(M);
  p.num_m = static_cast<int>((M + BM - 1) / BM);
  p.a_sf = A_sf;
  p.b_sf = B_sf;
  p.a_scale = a_scale;
  p.b_scale = b_scale;
  p.D = D;
  p.d_f32 = d_f32;
  p.status = status;
  const int64_t tiles = int64_t(p.num_m) * (N / BN);
  if (BN == 256) return launch<256>(ta, tb, p, tiles, s);
  return launch<128>(ta, tb, p, tiles, s);
}

}  // namespace nvfp4moe
