// NVFP4 W4A4 routed mixture-of-experts feed-forward layer: CPU ORACLE.
//
// This file is TEST INFRASTRUCTURE. Only the test-suite, the smoke check and the
// CPU-baseline leg of the benchmark load it. The product (the CUDA library under
// nvfp4_mixture_experts_w4a4_b200/csrc) never links, calls or includes it, and it
// includes nothing from the product.
//
// It is deliberately plain and slow: one obvious loop per definition, IEEE fp32 where
// the format fixes fp32 steps, fp64 everywhere else, no blocking or fusion.
//
// What the pages establish, and what is read into them
// -----------------------------------------------------
// * The routed experts are "NVFP4 W4A4": weights and activations both in NVFP4
//   (Qwen3.8-Flash-Next-NVFP4-SSD-Stream model card, "What this model is").
// * Two NVFP4 values share one packed byte (same card, "Why Hugging Face shows 68B
//   parameters and 8-bit precision").
// * The model has 512 routed experts; prefill batches up to 512 prompt tokens per
//   iteration to reuse the routed expert weights (Eider, "Qwen3.8 Flash Next" and
//   "Performance"); grouped routed prefill and routed decode are the kernels that
//   matter (Eider, "Development"; DwarfStar CUDA multi-GPU doc, grouped routed kernels).
// * The pages never define the NVFP4 arithmetic. This oracle uses the standard
//   definition: a value is e2m1(code) * e4m3(block scale) * fp32 tensor scale, with one
//   E4M3 block scale per 16 consecutive elements along K and the tensor scale of a
//   dynamically quantised tensor equal to amax / (6 * 448).
// * Readings taken where nothing fixes a step (the kernels take the same ones):
//   R1 E2M1 encode: round to nearest, ties to the even code, saturate at 6, keep the
//      sign (a negative value that rounds to zero encodes as 0x8).
//   R2 E4M3 encode: round to nearest even, saturate to +-448 (no NaN produced).
//   R3 block quantiser order: sf = e4m3(amax_b / (6*s_t)); inv = 1/(e4m3val(sf)*s_t);
//      code = e2m1(x*inv); every step one IEEE fp32 operation, round to nearest.
//   R4 element 2i of a row sits in the low nibble of byte i, element 2i+1 in the high.
//   R5 routing: top-k by descending logit, equal logits -> lower expert index first;
//      combine weights = softmax over the k selected logits.
//   R6 permutation: rows of expert e hold its (token, slot) pairs in ascending token
//      order; experts in ascending index.
//   R7 activations are quantised once per token with one tensor scale for the layer
//      input; the intermediate h of expert e is requantised with a per-expert tensor
//      scale s_h[e] that is given (or calibrated as amax_e(h) / 2688).
//   R8 SwiGLU: h = silu(g) * u with silu(g) = g / (1 + exp(-g)).
//   R9 combine: out[t] = sum over slots j = 0..k-1 (in order) of w[t][j] * y[t][j],
//      rounded once to bf16 (fp64 -> fp32 -> bf16, each round to nearest even).
//   R11 MXFP4 (the DwarfStar launcher's default format, read as the OCP microscaling
//      definition): E2M1 elements, one E8M0 scale 2^(E-127) per 32 consecutive elements
//      along K, no tensor scale; quantisation takes X = floor(log2(amax)) - 2 (2 = the
//      largest E2M1 exponent), clamped to [-127, 127], and codes e2m1(x / 2^X) (R1, so values
//      above 6 * 2^X saturate); an all-zero block gets E = 0.  Element packing as R4.
//      MXFP4 weights enter the NVFP4 layer exactly: a power of two 2^j is an E4M3 value for
//      j in [-9, 8], so each 16-element half of a block takes the E4M3 scale 2^(E-127-shift)
//      and the matrix the tensor scale 2^shift, shift = (largest E of a nonzero block) - 135;
//      a matrix whose nonzero blocks span more than 18 binades has no exact form (refused).
//   R12 shared expert (the SSD-Stream card's "shared experts ... remain BF16"; replicated
//      beside the routed experts in DwarfStar's expert-parallel pairs): a dense SwiGLU MLP
//      with bf16 weights, ys = Wd_s . bf16(silu(Wg_s x) * (Wu_s x)) for every token, x in bf16,
//      products and sums in fp64, its h rounded to bf16 (fp64 -> fp32 -> bf16); the layer's
//      output is bf16(routed + ys), one rounding of the fp64 sum.
//   R10 weight-only variant (W4A16; the NInfer card's "Limits" names NVFP4 weights without
//      an activation-quantisation site): x enters the gate/up products as bf16, the
//      intermediate h = silu(g) * u is rounded to bf16 (fp64 -> fp32 -> bf16) as the down
//      projection's activation, weights are dequantised NVFP4; products and sums in fp64.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fPIC -shared -pthread (see build.py).
// -ffp-contract=off keeps every fp32 step a separately rounded operation.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- E2M1 ----
// Code layout: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
// Exponent 0 is subnormal: value = mantissa * 0.5.  No Inf, no NaN.
double e2m1_value(int code) {
  const int s = (code >> 3) & 1;
  const int e = (code >> 1) & 3;
  const int m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// Reading R1: nearest representable magnitude; ties go to the even code; anything
// above 6 saturates to 6; the sign bit is copied from q (so -0.1 -> 0x8).
int e2m1_encode(float q) {
  const double a = std::fabs(static_cast<double>(q));
  if (a >= 6.0) return std::signbit(q) ? 15 : 7;  // saturate (also where |a - 6| rounds)
  int best = 0;
  double best_err = a;  // distance to code 0 (value 0)
  for (int c = 1; c < 8; ++c) {
    const double err = std::fabs(a - e2m1_value(c));
    if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      best_err = err;
    }
  }
  return std::signbit(q) ? (best | 8) : best;
}

// ---------------------------------------------------------------- E4M3 ----
// E4M3 "fn" variant: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.
// Exponent 0 is subnormal (m * 2^-9). 0x7F / 0xFF are NaN; max finite is 448 (0x7E).
double e4m3_value(int code) {
  const int s = (code >> 7) & 1;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  double mag;
  if (e == 15 && m == 7) {
    mag = NAN;
  } else if (e == 0) {
    mag = std::ldexp(static_cast<double>(m), -9);
  } else {
    mag = std::ldexp(1.0 + m / 8.0, e - 7);
  }
  return s ? -mag : mag;
}

// Reading R2: round to nearest, ties to even mantissa, clamp to 448.
// nearbyint() uses the default rounding mode, round-half-to-even.
int e4m3_encode(float v) {
  const int sign = std::signbit(v) ? 0x80 : 0;
  const double a = std::fabs(static_cast<double>(v));
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2;
  std::frexp(a, &e2);  // a = f * 2^e2, f in [0.5, 1)
  int E = e2 - 1;      // a = (2f) * 2^E, 2f in [1, 2)
  if (E < -6) {        // subnormal range: multiples of 2^-9
    const int m = static_cast<int>(std::nearbyint(std::ldexp(a, 9)));
    return sign | m;   // m == 8 is exactly the smallest normal, code 0x08
  }
  int m = static_cast<int>(std::nearbyint((std::ldexp(a, -E) - 1.0) * 8.0));
  if (m == 8) { m = 0; ++E; }
  int code = ((E + 7) << 3) | m;
  if (code > 0x7E) code = 0x7E;
  return sign | code;
}

// -------------------------------------------------------------- bf16 -------
float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// fp32 -> bf16, round to nearest even (finite inputs).
uint16_t float_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if (std::isnan(f)) return 0x7FC0;
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

// --------------------------------------------------------- quantiser -------
// Reading R3.  x is row-major [rows][K]; codes [rows][K/2] (R4), sf [rows][K/16].
void quantize_rows(const float* x, int64_t rows, int64_t K, float s_t, uint8_t* codes,
                   uint8_t* sf) {
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    const float* xr = x + r * K;
    for (int64_t b = 0; b < nb; ++b) {
      const float* xb = xr + b * 16;
      uint8_t* cb = codes + r * (K / 2) + b * 8;
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(xb[i]));
      int sfc = 0;
      if (s_t != 0.0f) {
        const float denom = 6.0f * s_t;
        const float ratio = amax / denom;
        sfc = e4m3_encode(ratio);
      }
      sf[r * nb + b] = static_cast<uint8_t>(sfc);
      const float sfv = static_cast<float>(e4m3_value(sfc));
      if (sfv == 0.0f) {
        std::memset(cb, 0, 8);
        continue;
      }
      const float scale = sfv * s_t;
      const float inv = 1.0f / scale;
      for (int i = 0; i < 8; ++i) {
        const float q0 = xb[2 * i] * inv;
        const float q1 = xb[2 * i + 1] * inv;
        cb[i] = static_cast<uint8_t>(e2m1_encode(q0) | (e2m1_encode(q1) << 4));
      }
    }
  }
}

float dynamic_scale(const float* x, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(x[i]));
  return amax / 2688.0f;  // 6 * 448 = 2688, exact in fp32
}

// --------------------------------------------------- exact block GEMM -------
// Twice an E2M1 value is an integer in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}.
// A 16-element block product sum(2a*2b) is therefore an exact integer, and
// sum * sf_a * sf_b / 4 is exact in fp64.
void decode_row_int(const uint8_t* codes, int64_t K, int8_t* out) {
  for (int64_t i = 0; i < K / 2; ++i) {
    out[2 * i] = static_cast<int8_t>(std::lround(2.0 * e2m1_value(codes[i] & 0xF)));
    out[2 * i + 1] = static_cast<int8_t>(std::lround(2.0 * e2m1_value(codes[i] >> 4)));
  }
}

// dot(a_row, b_row) of two quantised rows with their block scales (tensor scales not
// applied).  a_int / b_int are the integer-decoded rows, sfa / sfb the E4M3 codes.
double block_dot(const int8_t* a_int, const uint8_t* sfa, const int8_t* b_int,
                 const uint8_t* sfb, int64_t K) {
  double acc = 0.0;
  for (int64_t b = 0; b < K / 16; ++b) {
    int32_t isum = 0;
    for (int i = 0; i < 16; ++i) isum += int32_t(a_int[b * 16 + i]) * int32_t(b_int[b * 16 + i]);
    acc += static_cast<double>(isum) * e4m3_value(sfa[b]) * e4m3_value(sfb[b]) * 0.25;
  }
  return acc;
}

// Runs fn(i) for i in [0, n) on up to nthreads threads (dynamic work counter).
template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
  if (nthreads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  const int nt = static_cast<int>(std::min<int64_t>(nthreads, n));
  for (int t = 0; t < nt; ++t) {
    pool.emplace_back([&]() {
      for (;;) {
        const int64_t i = next.fetch_add(1);
        if (i >= n) break;
        fn(i);
      }
    });
  }
  for (auto& th : pool) th.join();
}

// ------------------------------------------------------- shared expert (R12) ----
// ys[t][n] for all T tokens: bf16 weights g, u [I][H] and d [H][I].
std::vector<double> shared_expert(const uint16_t* x_bf16, int64_t T, int64_t H, int64_t I, const uint16_t* g,
                                  const uint16_t* u, const uint16_t* d, int nth) {
  std::vector<double> ys(static_cast<size_t>(T * H), 0.0);
  parallel_for(T, nth, [&](int64_t t) {
    std::vector<double> h(static_cast<size_t>(I));
    for (int64_t i = 0; i < I; ++i) {
      double gv = 0.0, uv = 0.0;
      for (int64_t c = 0; c < H; ++c) {
        const double xv = bf16_to_float(x_bf16[t * H + c]);
        gv += xv * double(bf16_to_float(g[i * H + c]));
        uv += xv * double(bf16_to_float(u[i * H + c]));
      }
      h[size_t(i)] = double(bf16_to_float(float_to_bf16(static_cast<float>(gv / (1.0 + std::exp(-gv)) * uv))));
    }
    for (int64_t n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int64_t i = 0; i < I; ++i) acc += h[size_t(i)] * double(bf16_to_float(d[n * I + i]));
      ys[size_t(t * H + n)] = acc;
    }
  });
  return ys;
}

// ---------------------------------------------------------------- E8M0 ----
// Unsigned power-of-two scale: 2^(code - 127); 0xFF is NaN.
double e8m0_value(int code) { return code == 255 ? NAN : std::ldexp(1.0, code - 127); }

}  // namespace

extern "C" {

// ----------------------------------------------------------- codec API ------
double orc_e2m1_value(int code) { return e2m1_value(code & 15); }
int orc_e2m1_encode(float q) { return e2m1_encode(q); }
double orc_e4m3_value(int code) { return e4m3_value(code & 255); }
int orc_e4m3_encode(float v) { return e4m3_encode(v); }
uint16_t orc_float_to_bf16(float f) { return float_to_bf16(f); }

// Array forms of the encoders (same functions, one call per element).
void orc_e2m1_encode_n(const float* q, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<uint8_t>(e2m1_encode(q[i]));
}
void orc_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<uint8_t>(e4m3_encode(v[i]));
}

// Block quantiser (reading R3) on a row-major fp32 matrix.
// mode 0: tensor scale given in *tensor_scale; mode 1: dynamic, amax/2688, written back.
// sf is row-major [rows][K/16].  Returns 0, or -1 if K is not a multiple of 16.
int orc_quantize(const float* x, int64_t rows, int64_t K, int mode, float* tensor_scale,
                 uint8_t* codes, uint8_t* sf) {
  if (K % 16 != 0 || rows < 0) return -1;
  const float s_t = (mode == 1) ? dynamic_scale(x, rows * K) : *tensor_scale;
  *tensor_scale = s_t;
  quantize_rows(x, rows, K, s_t, codes, sf);
  return 0;
}

// Dequantise: v = e2m1(code) * e4m3(sf) * s_t, in fp64.
void orc_dequantize(const uint8_t* codes, const uint8_t* sf, float s_t, int64_t rows,
                    int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const int c = (k & 1) ? (byte >> 4) : (byte & 0xF);
      out[r * K + k] = e2m1_value(c) * e4m3_value(sf[r * (K / 16) + k / 16]) * double(s_t);
    }
}

// Quantised GEMM, C[m][n] = sum_k A[m][k] * B[n][k] * s_a * s_b, exact blocks, fp64.
void orc_gemm(const uint8_t* a_codes, const uint8_t* a_sf, float s_a, const uint8_t* b_codes,
              const uint8_t* b_sf, float s_b, int64_t M, int64_t N, int64_t K, double* out,
              int nthreads) {
  std::vector<int8_t> a_int(static_cast<size_t>(M * K)), b_int(static_cast<size_t>(N * K));
  for (int64_t m = 0; m < M; ++m) decode_row_int(a_codes + m * (K / 2), K, &a_int[m * K]);
  for (int64_t n = 0; n < N; ++n) decode_row_int(b_codes + n * (K / 2), K, &b_int[n * K]);
  parallel_for(M, nthreads, [&](int64_t m) {
    for (int64_t n = 0; n < N; ++n)
      out[m * N + n] = block_dot(&a_int[m * K], a_sf + m * (K / 16), &b_int[n * K],
                                 b_sf + n * (K / 16), K) *
                       double(s_a) * double(s_b);
  });
}

// Router, reading R5.  logits [T][E] -> ids [T][k], w [T][k].
void orc_route(const float* logits, int T, int E, int k, int32_t* ids, float* w) {
  std::vector<char> taken(static_cast<size_t>(E));
  for (int t = 0; t < T; ++t) {
    const float* l = logits + int64_t(t) * E;
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;  // strict: equal keeps lower index
      }
      taken[best] = 1;
      ids[int64_t(t) * k + j] = best;
    }
    const double l0 = l[ids[int64_t(t) * k]];
    double denom = 0.0;
    for (int j = 0; j < k; ++j) denom += std::exp(double(l[ids[int64_t(t) * k + j]]) - l0);
    for (int j = 0; j < k; ++j)
      w[int64_t(t) * k + j] =
          static_cast<float>(std::exp(double(l[ids[int64_t(t) * k + j]]) - l0) / denom);
  }
}

// Permutation, reading R6.  Returns 0, or -1 if an id is out of range.
// counts [E], offsets [E+1], row_token [T*k], row_slot [T*k], pair_to_row [T*k].
int orc_permute(const int32_t* ids, int T, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* row_token, int32_t* row_slot, int32_t* pair_to_row) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < int64_t(T) * k; ++p) {
    if (ids[p] < 0 || ids[p] >= E) return -1;
    counts[ids[p]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> fill(static_cast<size_t>(E), 0);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = ids[int64_t(t) * k + j];
      const int32_t row = offsets[e] + fill[e]++;
      row_token[row] = t;
      row_slot[row] = j;
      pair_to_row[int64_t(t) * k + j] = row;
    }
  return 0;
}

// The whole layer.  All pointers are host memory.  Weights are in the canonical
// (unpermuted, gate and up separate) layout with row-major block scales.
struct orc_moe_args {
  int32_t T, H, I, E, k;
  int32_t nthreads;
  const uint16_t* x_bf16;    // [T][H]
  const float* logits;       // [T][E]
  int32_t x_scale_mode;      // 0 given (*x_scale), 1 dynamic
  float* x_scale;            // in (given) / out
  const uint8_t* wg_codes;   // [E][I][H/2]
  const uint8_t* wg_sf;      // [E][I][H/16]
  const float* wg_scale;     // [E]
  const uint8_t* wu_codes;   // [E][I][H/2]
  const uint8_t* wu_sf;      // [E][I][H/16]
  const float* wu_scale;     // [E]
  const uint8_t* wd_codes;   // [E][H][I/2]
  const uint8_t* wd_sf;      // [E][H][I/16]
  const float* wd_scale;     // [E]
  int32_t h_scale_mode;      // 0 given (h_scale in), 1 calibrate (h_scale out)
  float* h_scale;            // [E]
  // outputs (required)
  uint16_t* out_bf16;        // [T][H]
  // optional outputs (nullable)
  double* out_f64;           // [T][H], before the bf16 rounding
  int32_t* ids;              // [T][k]
  float* w;                  // [T][k]
  int32_t* counts;           // [E]
  int32_t* offsets;          // [E+1]
  int32_t* row_token;        // [T*k]
  int32_t* row_slot;         // [T*k]
  int32_t* pair_to_row;      // [T*k]
  uint8_t* x_codes;          // [T][H/2]
  uint8_t* x_sf;             // [T][H/16]
  float* h_f32;              // [T*k][I], permuted rows
  uint8_t* h_codes;          // [T*k][I/2], permuted rows
  uint8_t* h_sf;             // [T*k][I/16]
  float* h_amax;             // [E]
  double* y_f64;             // [T*k][H], down-projection per permuted row, before w
  // optional shared expert (R12): shared_I = 0 for none; bf16 gate/up [I_s][H], down [H][I_s]
  int32_t shared_I;
  const uint16_t* shared_g;
  const uint16_t* shared_u;
  const uint16_t* shared_d;
};

int orc_moe_ffn(const orc_moe_args* a) {
  const int T = a->T, H = a->H, I = a->I, E = a->E, k = a->k;
  if (H % 16 || I % 16 || k < 1 || k > E || T < 0) return -1;
  const int64_t P = int64_t(T) * k;
  const int nth = std::max(1, int(a->nthreads));

  // 1. activation quantisation, once per token (R7)
  std::vector<float> xf(static_cast<size_t>(int64_t(T) * H));
  for (int64_t i = 0; i < int64_t(T) * H; ++i) xf[i] = bf16_to_float(a->x_bf16[i]);
  std::vector<uint8_t> xc(static_cast<size_t>(int64_t(T) * H / 2)), xs(static_cast<size_t>(int64_t(T) * H / 16));
  float s_x = (a->x_scale_mode == 1) ? dynamic_scale(xf.data(), int64_t(T) * H) : *a->x_scale;
  *a->x_scale = s_x;
  quantize_rows(xf.data(), T, H, s_x, xc.data(), xs.data());

  // 2. routing and permutation (R5, R6)
  std::vector<int32_t> ids(static_cast<size_t>(P)), counts(static_cast<size_t>(E)), offsets(static_cast<size_t>(E) + 1),
      row_token(static_cast<size_t>(P)), row_slot(static_cast<size_t>(P)), pair_to_row(static_cast<size_t>(P));
  std::vector<float> w(static_cast<size_t>(P));
  orc_route(a->logits, T, E, k, ids.data(), w.data());
  if (orc_permute(ids.data(), T, E, k, counts.data(), offsets.data(), row_token.data(),
                  row_slot.data(), pair_to_row.data()) != 0)
    return -2;

  // 3. gate/up GEMMs and SwiGLU (R8), per permuted row; h kept in fp32
  std::vector<float> h(static_cast<size_t>(P * I));
  std::vector<float> amax(static_cast<size_t>(E), 0.0f);
  parallel_for(E, nth, [&](int64_t e) {
    const int64_t n_e = counts[e];
    if (n_e == 0) return;
    std::vector<int8_t> wg_int(static_cast<size_t>(int64_t(I) * H)), wu_int(static_cast<size_t>(int64_t(I) * H)),
        x_int(static_cast<size_t>(H));
    const int64_t wofs = e * int64_t(I) * H;
    for (int64_t i = 0; i < I; ++i) {
      decode_row_int(a->wg_codes + (wofs + i * H) / 2, H, &wg_int[i * H]);
      decode_row_int(a->wu_codes + (wofs + i * H) / 2, H, &wu_int[i * H]);
    }
    float m = 0.0f;
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r) {
      const int t = row_token[r];
      decode_row_int(&xc[size_t(int64_t(t) * H / 2)], H, x_int.data());
      const uint8_t* xsf = &xs[size_t(int64_t(t) * H / 16)];
      for (int64_t i = 0; i < I; ++i) {
        const double g = block_dot(x_int.data(), xsf, &wg_int[i * H],
                                   a->wg_sf + (wofs + i * H) / 16, H) *
                         double(s_x) * double(a->wg_scale[e]);
        const double u = block_dot(x_int.data(), xsf, &wu_int[i * H],
                                   a->wu_sf + (wofs + i * H) / 16, H) *
                         double(s_x) * double(a->wu_scale[e]);
        const double silu = g / (1.0 + std::exp(-g));
        const float hv = static_cast<float>(silu * u);
        h[size_t(r * I + i)] = hv;
        m = std::max(m, std::fabs(hv));
      }
    }
    amax[e] = m;
  });

  // 4. per-expert requantisation scale (R7) and requantisation of h
  std::vector<float> s_h(static_cast<size_t>(E));
  for (int e = 0; e < E; ++e) {
    if (a->h_scale_mode == 1)
      s_h[e] = (counts[e] > 0) ? amax[e] / 2688.0f : 1.0f;
    else
      s_h[e] = a->h_scale[e];
    if (a->h_scale_mode == 1) a->h_scale[e] = s_h[e];
  }
  std::vector<uint8_t> hc(static_cast<size_t>(P * I / 2)), hs(static_cast<size_t>(P * I / 16));
  for (int e = 0; e < E; ++e) {
    const int64_t r0 = offsets[e], n_e = counts[e];
    quantize_rows(&h[size_t(r0 * I)], n_e, I, s_h[e], &hc[size_t(r0 * I / 2)],
                  &hs[size_t(r0 * I / 16)]);
  }

  // 5. down GEMM per permuted row
  std::vector<double> y(static_cast<size_t>(P * H));
  parallel_for(E, nth, [&](int64_t e) {
    if (counts[e] == 0) return;
    std::vector<int8_t> wd_int(static_cast<size_t>(int64_t(H) * I)), h_int(static_cast<size_t>(I));
    const int64_t wofs = e * int64_t(H) * I;
    for (int64_t n = 0; n < H; ++n) decode_row_int(a->wd_codes + (wofs + n * I) / 2, I, &wd_int[n * I]);
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r) {
      decode_row_int(&hc[size_t(r * I / 2)], I, h_int.data());
      const uint8_t* hsf = &hs[size_t(r * I / 16)];
      for (int64_t n = 0; n < H; ++n)
        y[size_t(r * H + n)] = block_dot(h_int.data(), hsf, &wd_int[n * I],
                                         a->wd_sf + (wofs + n * I) / 16, I) *
                               double(s_h[e]) * double(a->wd_scale[e]);
    }
  });

  // 6. weighted combine (R9), plus the shared expert (R12)
  std::vector<double> ys;
  if (a->shared_I > 0) ys = shared_expert(a->x_bf16, T, H, a->shared_I, a->shared_g, a->shared_u, a->shared_d, nth);
  for (int t = 0; t < T; ++t)
    for (int64_t n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) {
        const int64_t r = pair_to_row[size_t(int64_t(t) * k + j)];
        acc += double(w[size_t(int64_t(t) * k + j)]) * y[size_t(r * H + n)];
      }
      if (!ys.empty()) acc += ys[size_t(int64_t(t) * H + n)];
      if (a->out_f64) a->out_f64[int64_t(t) * H + n] = acc;
      a->out_bf16[int64_t(t) * H + n] = float_to_bf16(static_cast<float>(acc));
    }

  // optional outputs
  auto put = [](auto* dst, const auto& src) {
    if (dst) std::copy(src.begin(), src.end(), dst);
  };
  put(a->ids, ids);
  put(a->w, w);
  put(a->counts, counts);
  put(a->offsets, offsets);
  put(a->row_token, row_token);
  put(a->row_slot, row_slot);
  put(a->pair_to_row, pair_to_row);
  put(a->x_codes, xc);
  put(a->x_sf, xs);
  put(a->h_f32, h);
  put(a->h_codes, hc);
  put(a->h_sf, hs);
  put(a->h_amax, amax);
  put(a->y_f64, y);
  return 0;
}


// The weight-only (W4A16) layer, reading R10: routing, permutation and combine as in
// orc_moe_ffn; the expert products use dequantised weights and bf16 activations.
struct orc_moe_w4a16_args {
  int32_t T, H, I, E, k;
  int32_t nthreads;
  const uint16_t* x_bf16;    // [T][H]
  const float* logits;       // [T][E]
  const uint8_t* wg_codes;   // [E][I][H/2]
  const uint8_t* wg_sf;      // [E][I][H/16]
  const float* wg_scale;     // [E]
  const uint8_t* wu_codes;
  const uint8_t* wu_sf;
  const float* wu_scale;
  const uint8_t* wd_codes;   // [E][H][I/2]
  const uint8_t* wd_sf;      // [E][H][I/16]
  const float* wd_scale;     // [E]
  uint16_t* out_bf16;        // [T][H]
  // optional outputs (nullable)
  double* out_f64;           // [T][H], before the bf16 rounding
  int32_t* ids;              // [T][k]
  float* w;                  // [T][k]
  int32_t* counts;           // [E]
  int32_t* offsets;          // [E+1]
  int32_t* row_token;        // [T*k]
  int32_t* pair_to_row;      // [T*k]
  uint16_t* h_bf16;          // [T*k][I], permuted rows
  double* y_f64;             // [T*k][H], down projection per permuted row, before w
  int32_t shared_I;          // optional shared expert (R12), as in orc_moe_args
  const uint16_t* shared_g;
  const uint16_t* shared_u;
  const uint16_t* shared_d;
};

namespace {
// Row r of an NVFP4 matrix with K columns as doubles: e2m1(code) * e4m3(sf) * s.
void dequant_row(const uint8_t* codes, const uint8_t* sf, double s, int64_t r, int64_t K, double* out) {
  for (int64_t c = 0; c < K; ++c) {
    const int byte = codes[(r * K + c) / 2];
    const int code = (c & 1) ? (byte >> 4) : (byte & 15);
    out[c] = e2m1_value(code) * e4m3_value(sf[(r * K + c) / 16]) * s;
  }
}
}  // namespace

int orc_moe_ffn_w4a16(const orc_moe_w4a16_args* a) {
  const int T = a->T, H = a->H, I = a->I, E = a->E, k = a->k;
  if (H % 16 || I % 16 || k < 1 || k > E || T < 0) return -1;
  const int64_t P = int64_t(T) * k;
  const int nth = std::max(1, int(a->nthreads));

  // 1. routing and permutation (R5, R6)
  std::vector<int32_t> ids(static_cast<size_t>(P)), counts(static_cast<size_t>(E)), offsets(static_cast<size_t>(E) + 1),
      row_token(static_cast<size_t>(P)), row_slot(static_cast<size_t>(P)), pair_to_row(static_cast<size_t>(P));
  std::vector<float> w(static_cast<size_t>(P));
  orc_route(a->logits, T, E, k, ids.data(), w.data());
  if (orc_permute(ids.data(), T, E, k, counts.data(), offsets.data(), row_token.data(), row_slot.data(),
                  pair_to_row.data()) != 0)
    return -2;

  // 2. gate/up with bf16 x and dequantised weights, SwiGLU (R8), h rounded to bf16 (R10)
  std::vector<uint16_t> h(static_cast<size_t>(P * I));
  parallel_for(E, nth, [&](int64_t e) {
    if (counts[e] == 0) return;
    std::vector<double> wg(static_cast<size_t>(int64_t(I) * H)), wu(static_cast<size_t>(int64_t(I) * H)),
        x(static_cast<size_t>(H));
    for (int64_t i = 0; i < I; ++i) {
      dequant_row(a->wg_codes, a->wg_sf, a->wg_scale[e], e * I + i, H, &wg[size_t(i * H)]);
      dequant_row(a->wu_codes, a->wu_sf, a->wu_scale[e], e * I + i, H, &wu[size_t(i * H)]);
    }
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r) {
      const int t = row_token[r];
      for (int64_t c = 0; c < H; ++c) x[size_t(c)] = bf16_to_float(a->x_bf16[int64_t(t) * H + c]);
      for (int64_t i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < H; ++c) {
          g += x[size_t(c)] * wg[size_t(i * H + c)];
          u += x[size_t(c)] * wu[size_t(i * H + c)];
        }
        const double hv = g / (1.0 + std::exp(-g)) * u;
        h[size_t(r * I + i)] = float_to_bf16(static_cast<float>(hv));
      }
    }
  });

  // 3. down projection per permuted row
  std::vector<double> y(static_cast<size_t>(P * H));
  parallel_for(E, nth, [&](int64_t e) {
    if (counts[e] == 0) return;
    std::vector<double> wd(static_cast<size_t>(int64_t(H) * I));
    for (int64_t n = 0; n < H; ++n) dequant_row(a->wd_codes, a->wd_sf, a->wd_scale[e], e * H + n, I, &wd[size_t(n * I)]);
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r)
      for (int64_t n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i) acc += double(bf16_to_float(h[size_t(r * I + i)])) * wd[size_t(n * I + i)];
        y[size_t(r * H + n)] = acc;
      }
  });

  // 4. weighted combine (R9), plus the shared expert (R12)
  std::vector<double> ys;
  if (a->shared_I > 0) ys = shared_expert(a->x_bf16, T, H, a->shared_I, a->shared_g, a->shared_u, a->shared_d, nth);
  for (int t = 0; t < T; ++t)
    for (int64_t n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) {
        const int64_t r = pair_to_row[size_t(int64_t(t) * k + j)];
        acc += double(w[size_t(int64_t(t) * k + j)]) * y[size_t(r * H + n)];
      }
      if (!ys.empty()) acc += ys[size_t(int64_t(t) * H + n)];
      if (a->out_f64) a->out_f64[int64_t(t) * H + n] = acc;
      a->out_bf16[int64_t(t) * H + n] = float_to_bf16(static_cast<float>(acc));
    }

  auto put = [](auto* dst, const auto& src) {
    if (dst) std::copy(src.begin(), src.end(), dst);
  };
  put(a->ids, ids);
  put(a->w, w);
  put(a->counts, counts);
  put(a->offsets, offsets);
  put(a->row_token, row_token);
  put(a->pair_to_row, pair_to_row);
  put(a->h_bf16, h);
  put(a->y_f64, y);
  return 0;
}


// ---------------------------------------------------------------- MXFP4 (R11) ----
double orc_e8m0_value(int code) { return e8m0_value(code & 255); }

// Quantises rows x K fp32 values to MXFP4: codes [rows][K/2], e8m0 [rows][K/32].
int orc_mx_quantize(const float* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* e8m0) {
  if (K % 32 != 0 || rows < 0) return -1;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) {
      const float* v = x + r * K + b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(v[i]));
      int X = -127;
      if (amax > 0.0f) {
        int e = 0;
        std::frexp(static_cast<double>(amax), &e);  // amax = m 2^e, m in [0.5, 1): floor(log2) = e - 1
        X = std::min(127, std::max(-127, e - 1 - 2));
      }
      e8m0[r * (K / 32) + b] = static_cast<uint8_t>(X + 127);
      for (int i = 0; i < 32; ++i) {
        const float q = static_cast<float>(std::ldexp(static_cast<double>(v[i]), -X));  // exact
        const int c = e2m1_encode(q);
        const int64_t k = b * 32 + i;
        uint8_t& byte = codes[r * (K / 2) + k / 2];
        byte = (k & 1) ? static_cast<uint8_t>((byte & 0x0F) | (c << 4)) : static_cast<uint8_t>((byte & 0xF0) | c);
      }
    }
  return 0;
}

// v = e2m1(code) * 2^(E - 127), in fp64.
void orc_mx_dequantize(const uint8_t* codes, const uint8_t* e8m0, int64_t rows, int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const int c = (k & 1) ? (byte >> 4) : (byte & 0xF);
      out[r * K + k] = e2m1_value(c) * e8m0_value(e8m0[r * (K / 32) + k / 32]);
    }
}

// The NVFP4 form of an MXFP4 matrix (R11): the codes are unchanged; writes the row-major
// E4M3 block scales sf [rows][K/16] and the tensor scale.  Returns -3 when the nonzero
// blocks span more than 18 binades.
int orc_mx_to_nvfp4(const uint8_t* codes, const uint8_t* e8m0, int64_t rows, int64_t K, uint8_t* sf,
                    float* tensor_scale) {
  if (K % 32 != 0 || rows < 0) return -1;
  auto nonzero = [&](int64_t r, int64_t b) {
    for (int i = 0; i < 16; ++i)
      if (codes[r * (K / 2) + b * 16 + i] & 0x77) return true;  // a nonzero magnitude nibble
    return false;
  };
  int emax = -1;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b)
      if (nonzero(r, b)) emax = std::max(emax, int(e8m0[r * (K / 32) + b]));
  const int shift = emax < 0 ? 0 : emax - 127 - 8;
  *tensor_scale = static_cast<float>(std::ldexp(1.0, shift));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) {
      uint8_t code = 0;
      if (nonzero(r, b)) {
        const int j = int(e8m0[r * (K / 32) + b]) - 127 - shift;
        if (j < -9) return -3;
        code = static_cast<uint8_t>(e4m3_encode(static_cast<float>(std::ldexp(1.0, j))));
      }
      sf[r * (K / 16) + 2 * b] = code;
      sf[r * (K / 16) + 2 * b + 1] = code;
    }
  return 0;
}

}  // extern "C"
