// Test-only kernel: runs the flash kernel's FMA-pipe 2^x routine
// (exp2_poly2 in the library's sm100.cuh) and the MUFU instruction beside it
// on given inputs, so that the tests can check the routine on the device.
#include "sm100.cuh"

__global__ void exp2_poly_probe(const float* x, float* y_poly, float* y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n) return;
  float a, b;
  sdattn::exp2_poly2(x[i], x[i + 1], a, b);
  y_poly[i] = a;
  y_poly[i + 1] = b;
  y_mufu[i] = sdattn::ex2_approx(x[i]);
  y_mufu[i + 1] = sdattn::ex2_approx(x[i + 1]);
}

extern "C" int exp2_poly_probe_run(const float* x, float* y_poly, float* y_mufu, int n) {
  exp2_poly_probe<<<(n / 2 + 255) / 256, 256>>>(x, y_poly, y_mufu, n);
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 1;
}
