// Host driver for the library's block quantiser codes and packing (the same source the
// encode and decode kernels compile for the device): reads blocks of 16 fp32 values and a
// bit-width b from stdin; for each block writes lo, step (fp32), the 16 codes (uint8), the
// 2 b packed bytes (padded to 16) and the 16 codes unpacked from those bytes (uint8).
#include <cstdio>
#include <cstring>

#include "fp16_exact.cuh"

int main() {
  int b = 0;
  if (fread(&b, sizeof(int), 1, stdin) != 1 || b < 1 || b > 8) return 1;
  const float flev = (float)((1 << b) - 1);
  float v[16];
  while (fread(v, sizeof(float), 16, stdin) == 16) {
    float mn = v[0], mx = v[0];
    for (int j = 1; j < 16; ++j) {
      mn = fminf(mn, v[j]);
      mx = fmaxf(mx, v[j]);
    }
    const float lo = jolt::rd16(mn);
    const float step = jolt::quant_step(mx, lo, flev, 1.0f / flev);
    const float inv = (step > 0.f && step <= jolt::kFp16Max) ? 1.0f / step : 0.f;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    unsigned char codes[16], bytes[16], back[16];
    for (int j = 0; j < 16; ++j) {
      const uint32_t c = jolt::block_code(v[j], lo, inv, flev);
      codes[j] = (unsigned char)c;
      jolt::pack_code(w, j, b, c);
    }
    memset(bytes, 0, sizeof bytes);
    for (int i = 0; i < 2 * b; ++i) bytes[i] = (unsigned char)(w[i >> 2] >> ((i & 3) * 8));
    uint32_t r[4] = {0u, 0u, 0u, 0u};
    for (int i = 0; i < 2 * b; ++i) r[i >> 2] |= (uint32_t)bytes[i] << ((i & 3) * 8);
    for (int j = 0; j < 16; ++j) back[j] = (unsigned char)jolt::unpack_code(r, j, b);
    fwrite(&lo, sizeof(float), 1, stdout);
    fwrite(&step, sizeof(float), 1, stdout);
    fwrite(codes, 1, 16, stdout);
    fwrite(bytes, 1, 16, stdout);
    fwrite(back, 1, 16, stdout);
  }
  return 0;
}
