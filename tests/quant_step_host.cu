// Host driver for the library's exact fp16 helpers (the same source the table and encode
// kernels compile for the device): reads (block minimum, block maximum) pairs as fp32 from
// stdin, writes lo = rd16(min), quant_step(max, lo) for b = 1, 2, 3, 4, 8, the branch-free
// quant_step_sel and the bracketed quant_step_cvt for the same b, as fp32.
#include <cstdio>
#include <vector>

#include "fp16_exact.cuh"

int main() {
  const int bits[5] = {1, 2, 3, 4, 8};
  std::vector<float> in;
  float v[2];
  while (fread(v, sizeof(float), 2, stdin) == 2) {
    in.push_back(v[0]);
    in.push_back(v[1]);
  }
  for (size_t i = 0; i < in.size(); i += 2) {
    float out[16];
    out[0] = jolt::rd16(in[i]);
    for (int j = 0; j < 5; ++j) {
      const float flev = (float)((1 << bits[j]) - 1);
      out[1 + j] = jolt::quant_step(in[i + 1], out[0], flev, 1.0f / flev);
      out[6 + j] = jolt::quant_step_sel(in[i + 1], out[0], flev, 1.0f / flev);
      out[11 + j] = jolt::quant_step_cvt(in[i + 1], out[0], bits[j]);
    }
    fwrite(out, sizeof(float), 16, stdout);
  }
  return 0;
}
