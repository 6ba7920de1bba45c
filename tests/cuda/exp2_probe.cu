// Test probe (built by tests/test_gpu_exp2.py): evaluates the stream kernel's
// FMA-pipe 2^x (ex2_fma_pair) and the special-function unit's ex2.approx on
// the same arguments, so that the test can compare both with exact powers.
#include "../../speculative_decoding_verification_94_b200/csrc/sv_stream.cuh"

__global__ void exp2_probe_kernel(const float* x, float* y_fma, float* y_sfu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  float pa, pb;
  sv::f2_unpack(sv::ex2_fma_pair(a, b), pa, pb);
  y_fma[i] = pa;
  y_sfu[i] = sv::ex2(a);
  if (i + 1 < n) {
    y_fma[i + 1] = pb;
    y_sfu[i + 1] = sv::ex2(b);
  }
}

extern "C" int exp2_probe(const float* x, float* y_fma, float* y_sfu, int n) {
  if (n <= 0) return 0;
  const int pairs = (n + 1) / 2;
  exp2_probe_kernel<<<(pairs + 255) / 256, 256>>>(x, y_fma, y_sfu, n);
  return (int)cudaDeviceSynchronize();
}

// The float64 powers of the sampling-tree kernel: the Taylor form and the
// table-assisted form (table filled as the kernel fills it).
__global__ void exp2d_probe_kernel(const double* x, double* y_tab, double* y_taylor, int n) {
  __shared__ double t16[16];
  if (threadIdx.x < 16) t16[threadIdx.x] = sv::exp2_f64((double)threadIdx.x * 0.0625);
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  y_tab[i] = sv::exp2_f64_tab(x[i], t16);
  y_taylor[i] = sv::exp2_f64(x[i]);
}

extern "C" int exp2d_probe(const double* x, double* y_tab, double* y_taylor, int n) {
  if (n <= 0) return 0;
  exp2d_probe_kernel<<<(n + 255) / 256, 256>>>(x, y_tab, y_taylor, n);
  return (int)cudaDeviceSynchronize();
}
