// Host-side conversions from the CUDA toolkit headers (cuda_fp4.h, cuda_fp8.h), used as an
// independent library pin for the oracle's E2M1 / E4M3 encoders.
// Reads fp32 values (binary) from stdin, writes e2m1 code then e4m3 satfinite code per value.
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cstdio>
#include <vector>

int main() {
  std::vector<float> v;
  float f;
  while (std::fread(&f, 4, 1, stdin) == 1) v.push_back(f);
  for (float x : v) {
    unsigned char out[2];
    out[0] = static_cast<unsigned char>(__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest));
    out[1] = static_cast<unsigned char>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
    std::fwrite(out, 1, 2, stdout);
  }
  return 0;
}
