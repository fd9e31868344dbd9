// Throughput probe (a stand-alone executable, not part of the library).
//
// Measures, per SM per clock: exp2 results on the MUFU (ex2.approx, in fp32 and on packed
// f16 / bf16 pairs) and on the FMA pipe (the packed-pair polynomial the selector uses for
// part of its exponentials); and fp64
// additions of bf16 values widened to double (by conversion, or built from the bits with
// integer operations), the inner step of the selector's exact means.  148 CTAs of W warps
// each run independent chains; only a per-CTA clock count and one value per thread are
// written.
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

// Packed half-precision exponentials: each ex2.approx on a .f16x2 / .bf16x2 register gives two
// results; the chain stays packed (one fma.rn on the pair feeds the next exponential).
template <bool BF16, int ILP>
__global__ void exp_probe_x2(uint32_t* out, int iters, uint32_t a, uint32_t b, long long* cyc) {
  uint32_t x[ILP];
  for (int i = 0; i < ILP; ++i) x[i] = 0x3c003c00u ^ ((threadIdx.x + i) & 7);
  const long long t0 = clock64();
  for (int n = 0; n < iters; ++n) {
#pragma unroll
    for (int i = 0; i < ILP; ++i) {
      uint32_t y;
      if (BF16) {
        asm volatile("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(y) : "r"(x[i]), "r"(a), "r"(b));
        asm volatile("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(x[i]) : "r"(y));
      } else {
        asm volatile("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(y) : "r"(x[i]), "r"(a), "r"(b));
        asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(x[i]) : "r"(y));
      }
    }
  }
  const long long t1 = clock64();
  uint32_t s = 0;
  for (int i = 0; i < ILP; ++i) s ^= x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <bool BF16, int ILP>
void run_x2(int warps, uint32_t* out, long long* cyc) {
  const int iters = 2000;
  // a = 0.5 and b = -0.3 in each half
  const uint32_t a = BF16 ? 0x3f003f00u : 0x38003800u, b = BF16 ? 0xbe9abe9au : 0xb4cdb4cdu;
  for (int rep = 0; rep < 2; ++rep) exp_probe_x2<BF16, ILP><<<148, warps * 32>>>(out, iters, a, b, cyc);
  cudaDeviceSynchronize();
  long long h[148];
  cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
  double mx = 0;
  for (int i = 0; i < 148; ++i) mx = h[i] > mx ? (double)h[i] : mx;
  printf("%s ilp=%2d warps/SM=%2d: %.2f exp2 per clock per SM (two per instruction)\n",
         BF16 ? "mufu bf16x2" : "mufu f16x2", ILP, warps, (double)warps * 32 * iters * ILP * 2 / mx);
}

template <int MODE>
__global__ void f64_probe(const uint32_t* in, double* out, int iters, long long* cyc) {
  uint32_t w[8];
  for (int i = 0; i < 8; ++i) w[i] = in[(threadIdx.x + i * 37) & 1023] | 0x3f803f80u;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const long long t0 = clock64();
  for (int n = 0; n < iters; ++n) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t x = w[i] + n;  // upper half: a normal bf16
      double d;
      if (MODE == 0) {
        d = (double)__uint_as_float(x & 0xffff0000u);
      } else {  // sign | (exponent + 1023 - 127, mantissa) in the high word
        d = __hiloint2double((int)((((x >> 3) & 0x0FFFE000u) + 0x38000000u) | (x & 0x80000000u)), 0);
      }
      acc[i] += d;
    }
  }
  const long long t1 = clock64();
  double s = 0.0;
  for (int i = 0; i < 8; ++i) s += acc[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int MODE>
void run_f64(int warps, const uint32_t* in, double* out, long long* cyc) {
  const int iters = 1000;
  for (int rep = 0; rep < 2; ++rep) f64_probe<MODE><<<148, warps * 32>>>(in, out, iters, cyc);
  cudaDeviceSynchronize();
  long long h[148];
  cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
  double mx = 0;
  for (int i = 0; i < 148; ++i) mx = h[i] > mx ? (double)h[i] : mx;
  printf("fp64 add of bf16 (%s) warps/SM=%2d: %.2f per clock per SM\n", MODE ? "built from bits" : "converted",
         warps, (double)warps * 32 * iters * 8 / mx);
}

int main() {
  float* out;
  long long* cyc;
  cudaMalloc(&out, 148 * 1024 * 4);  // 148 CTAs x at most 32 warps x 32 threads
  cudaMalloc(&cyc, 148 * 8);
  for (int w : {4, 8, 16, 32}) { run<0, 8>(w, out, cyc); run<0, 16>(w, out, cyc); }
  for (int w : {4, 8, 16, 32}) { run<1, 8>(w, out, cyc); run<1, 16>(w, out, cyc); }
  for (int w : {4, 8, 16, 32}) {
    run_x2<false, 8>(w, reinterpret_cast<uint32_t*>(out), cyc);
    run_x2<true, 8>(w, reinterpret_cast<uint32_t*>(out), cyc);
  }
  uint32_t* in;
  double* out64;
  cudaMalloc(&in, 1024 * 4);
  cudaMemset(in, 0, 1024 * 4);
  cudaMalloc(&out64, 148 * 1024 * 8);
  for (int w : {8, 16, 32}) { run_f64<0>(w, in, out64, cyc); run_f64<1>(w, in, out64, cyc); }
  const cudaError_t e = cudaGetLastError();
  printf("status: %s\n", cudaGetErrorString(e));
  return e == cudaSuccess ? 0 : 1;
}
