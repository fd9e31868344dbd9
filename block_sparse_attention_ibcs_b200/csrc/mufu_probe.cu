// Exponential throughput probe (a stand-alone executable, not part of the library).
//
// Measures exp2 results per SM per clock on the MUFU (ex2.approx) and on the FMA pipe
// (the packed-pair polynomial the selector uses for part of its exponentials), with
// 148 CTAs of W warps each running ILP independent chains; only a per-CTA clock count and
// one float per thread are written.  Used to set the selector's exponential bound.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

template <int MODE, int ILP>
__global__ void exp_probe(float* out, int iters, float a, float b, long long* cyc) {
  float x[ILP];
  for (int i = 0; i < ILP; ++i) x[i] = 0.001f * (threadIdx.x + i);
  const long long t0 = clock64();
  for (int n = 0; n < iters; ++n) {
#pragma unroll
    for (int i = 0; i < ILP; i += 2) {
      const float y0 = fmaf(x[i], a, b), y1 = fmaf(x[i + 1], a, b);
      if (MODE == 0) {
        x[i] = fast_exp2(y0);
        x[i + 1] = fast_exp2(y1);
      } else {
        const float2 r = f2_unpack(exp2_poly_x2(y0, y1));
        x[i] = r.x;
        x[i + 1] = r.y;
      }
    }
  }
  const long long t1 = clock64();
  float s = 0.f;
  for (int i = 0; i < ILP; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int MODE, int ILP>
void run(int warps, float* out, long long* cyc) {
  const int iters = 2000;
  for (int rep = 0; rep < 2; ++rep) exp_probe<MODE, ILP><<<148, warps * 32>>>(out, iters, 0.5f, -0.3f, cyc);
  cudaDeviceSynchronize();
  long long h[148];
  cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
  double mx = 0;
  for (int i = 0; i < 148; ++i) mx = h[i] > mx ? (double)h[i] : mx;
  printf("%s ilp=%2d warps/SM=%2d: %.2f exp2 per clock per SM\n", MODE ? "poly" : "mufu", ILP, warps,
         (double)warps * 32 * iters * ILP / mx);
}

int main() {
  float* out;
  long long* cyc;
  cudaMalloc(&out, 148 * 1024 * 4);  // 148 CTAs x at most 32 warps x 32 threads
  cudaMalloc(&cyc, 148 * 8);
  for (int w : {4, 8, 16, 32}) { run<0, 8>(w, out, cyc); run<0, 16>(w, out, cyc); }
  for (int w : {4, 8, 16, 32}) { run<1, 8>(w, out, cyc); run<1, 16>(w, out, cyc); }
  const cudaError_t e = cudaGetLastError();
  printf("status: %s\n", cudaGetErrorString(e));
  return e == cudaSuccess ? 0 : 1;
}
