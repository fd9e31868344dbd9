// Gather-bandwidth probe: how fast can one B200 SM pull 4-token K/V blocks (4 rows x
// 256 B = 1 KB, the unit the packed attention gathers) from an L2-resident buffer into
// shared memory?  This sets the ceiling the attention kernel is measured against.
//
//   cpasync : 16-byte cp.async per thread (the attention kernel's copy), 8 warps, one
//             32 KB tile in flight per CTA
//   bulk<NT>: 1 KB cp.async.bulk copies completing on an mbarrier, NT tiles in flight
//   pipe<NST>: the attention kernel's pattern: 4 to 16 warps, K and V of a 128-token tile
//             per 64 KB stage, NST stages in flight, footprints of 16, 40 and 64 MB
//
// Prints cycles per 32 KB tile, bytes/cycle per SM and in aggregate, for grids of 148
// (one CTA per SM), 74 and 37 CTAs.  Block indices come from a fixed LCG; every address
// stays inside the 64 MB buffer and every wait is bounded.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <vector>

namespace {

__device__ __forceinline__ uint32_t sa(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__global__ void gather_cpasync(const uint8_t* __restrict__ g, const int* __restrict__ blocks, int nb,
                               int iters, long long* out) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sbase = sa(sm);
  const int tid = threadIdx.x;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    for (int c = tid; c < 2048; c += blockDim.x) {
      const int r = c >> 4, u = c & 15;
      const int blk = blocks[((blockIdx.x * iters + it) * 32 + (r >> 2)) % nb];
      const uint8_t* src = g + ((size_t)blk * 4 + (r & 3)) * 256 + u * 16;
      const uint32_t dst = sbase + (u >> 3) * 16384 + r * 128 + (((u & 7) ^ (r & 7)) << 4);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }
  if (tid == 0) out[blockIdx.x] = clock64() - t0;
}

template <int NT>
__global__ void gather_bulk(const uint8_t* __restrict__ g, const int* __restrict__ blocks, int nb,
                            int iters, long long* out, int* err) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ __align__(8) uint64_t bar[NT];
  const int tid = threadIdx.x;  // one warp: lane l copies block l of each tile
  if (tid == 0) {
    for (int i = 0; i < NT; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sa(&bar[i])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int it) {
    const int st = it % NT;
    if (tid == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa(&bar[st])), "r"(32768)
                   : "memory");
    __syncwarp();
    const int blk = blocks[((blockIdx.x * iters + it) * 32 + tid) % nb];
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 1024, [%2];" ::"r"(
            sa(sm) + st * 32768 + tid * 1024),
        "l"(g + (size_t)blk * 1024), "r"(sa(&bar[st]))
        : "memory");
  };
  const long long t0 = clock64();
  for (int it = 0; it < NT && it < iters; ++it) issue(it);
  for (int it = 0; it < iters; ++it) {
    const int st = it % NT;
    uint32_t ok = 0;
    for (long long k = 0; k < 20000000 && !ok; ++k)
      asm volatile(
          "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0,1,0,p; }"
          : "=r"(ok)
          : "r"(sa(&bar[st])), "r"((it / NT) & 1)
          : "memory");
    if (!ok && tid == 0) atomicExch(err, 1);
    __syncwarp();
    if (it + NT < iters) issue(it + NT);
  }
  if (tid == 0) out[blockIdx.x] = clock64() - t0;
}

// The attention kernel's own pattern: W copying warps; a stage is one 128-token tile of K
// and of V (the same 32 block indices into a K half and a V half of a footprint of F bytes,
// 64 KB per stage); NST stages in flight (cp.async groups), so the copy rate rather than one
// tile's latency is measured.  As in the kernel, each warp loads a tile's 32 block indices
// with one coalesced load a tile ahead and hands them to the copying lanes by shuffles; the
// random words map into the footprint by a multiply-high.
template <int NST, int EXTRA = 0>
__global__ void gather_pipe(const uint8_t* __restrict__ g, const uint32_t* __restrict__ blocks, int nb,
                            int iters, size_t half_bytes, long long* out, uint32_t zero = 0) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sbase = sa(sm);
  const int tid = threadIdx.x, lane = tid & 31;
  const int nthr = blockDim.x;
  const uint32_t nblk = (uint32_t)(half_bytes / 1024);
  const int per_thread = (4096 + nthr - 1) / nthr;  // warp-uniform trip count
  uint32_t cur = blocks[(blockIdx.x * iters * 32 + lane) & (nb - 1)];
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    const uint32_t nxt = blocks[((blockIdx.x * iters + it + 1) * 32 + lane) & (nb - 1)];
    const uint32_t stage = sbase + (uint32_t)(it % NST) * 65536u;
    for (int k = 0; k < per_thread; ++k) {
      const int c = tid + k * nthr;
      const int kv = (c >> 11) & 1, r = (c >> 4) & 127, u = c & 15;
      uint32_t blk = __umulhi(__shfl_sync(0xffffffffu, cur, r >> 2), nblk);
#pragma unroll
      for (int x = 0; x < EXTRA; ++x)  // EXTRA integer instructions per copy (zero is 0)
        asm volatile("xor.b32 %0, %0, %1;" : "+r"(blk) : "r"(zero));
      if (c < 4096) {
        const uint8_t* src = g + (size_t)kv * half_bytes + ((size_t)blk * 4 + (r & 3)) * 256 + u * 16;
        const uint32_t dst = stage + kv * 32768u + (u >> 3) * 16384 + r * 128 + (((u & 7) ^ (r & 7)) << 4);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      }
    }
    cur = nxt;
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" ::"n"(NST - 1) : "memory");
    __syncthreads();
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (tid == 0) out[blockIdx.x] = clock64() - t0;
}

}  // namespace

int main() {
  const size_t G = 64ull << 20;
  const int nblocks = (int)(G / 1024);
  uint8_t* g = nullptr;
  int* blocks = nullptr;
  long long* out = nullptr;
  int* err = nullptr;
  if (cudaMalloc(&g, G) != cudaSuccess) return 1;
  cudaMemset(g, 1, G);
  std::vector<int> hb(1 << 20);
  uint32_t x = 12345;
  for (auto& b : hb) {
    x = x * 1664525u + 1013904223u;
    b = (int)(x % (uint32_t)nblocks);
  }
  cudaMalloc(&blocks, hb.size() * 4);
  cudaMemcpy(blocks, hb.data(), hb.size() * 4, cudaMemcpyHostToDevice);
  cudaMalloc(&out, 148 * 8);
  cudaMalloc(&err, 4);
  cudaMemset(err, 0, 4);
  const int iters = 64;  // (147*64 + 63)*32 + 31 < 2^20 entries
  auto report = [&](const char* name, int grid) {
    cudaDeviceSynchronize();
    std::vector<long long> h(grid);
    cudaMemcpy(h.data(), out, grid * 8, cudaMemcpyDeviceToHost);
    double avg = 0;
    for (auto v : h) avg += (double)v;
    avg /= grid;
    printf("grid %3d %-10s %7.0f cycles/32KB tile  %5.1f B/cycle/SM  aggregate %6.0f B/cycle\n", grid, name,
           avg / iters, 32768.0 * iters / avg, grid * 32768.0 * iters / avg);
  };
  cudaFuncSetAttribute(gather_cpasync, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * 1024);
  cudaFuncSetAttribute(gather_bulk<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 32 * 1024);
  cudaFuncSetAttribute(gather_bulk<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
  for (int grid : {148, 74, 37}) {
    for (int rep = 0; rep < 2; ++rep) gather_cpasync<<<grid, 256, 33 * 1024>>>(g, blocks, (int)hb.size(), iters, out);
    report("cpasync", grid);
    for (int rep = 0; rep < 2; ++rep) gather_bulk<1><<<grid, 32, 32 * 1024>>>(g, blocks, (int)hb.size(), iters, out, err);
    report("bulk x1", grid);
    for (int rep = 0; rep < 2; ++rep) gather_bulk<4><<<grid, 32, 128 * 1024>>>(g, blocks, (int)hb.size(), iters, out, err);
    report("bulk x4", grid);
  }
  // the attention pattern: K+V stages of 64 KB, footprints from 16 MB to the whole 64 MB,
  // 4 to 16 copying warps
  std::vector<uint32_t> hr(1u << 20);
  for (auto& v : hr) v = (x = x * 1664525u + 1013904223u);
  uint32_t* rnd;
  cudaMalloc(&rnd, hr.size() * 4);
  cudaMemcpy(rnd, hr.data(), hr.size() * 4, cudaMemcpyHostToDevice);
  cudaFuncSetAttribute(gather_pipe<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(gather_pipe<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
  for (size_t mb : {16, 40, 64}) {
    const size_t half = (mb << 20) / 2;
    for (int warps : {4, 7, 12, 16}) {
      auto report_pipe = [&](const char* name) {
        cudaDeviceSynchronize();
        std::vector<long long> h(148);
        cudaMemcpy(h.data(), out, 148 * 8, cudaMemcpyDeviceToHost);
        double avg = 0;
        for (auto v : h) avg += (double)v;
        avg /= 148;
        printf("footprint %2zu MB %2d warps %-8s %7.0f cycles/64KB stage  %5.1f B/cycle/SM  aggregate %6.0f B/cycle\n",
               mb, warps, name, avg / iters, 65536.0 * iters / avg, 148 * 65536.0 * iters / avg);
      };
      if (mb == 40) {
        for (int rep = 0; rep < 2; ++rep)
          gather_pipe<1><<<148, warps * 32, 64 * 1024>>>(g, rnd, (int)hr.size(), iters, half, out);
        report_pipe("pipe x1");
      }
      for (int rep = 0; rep < 2; ++rep)
        gather_pipe<3><<<148, warps * 32, 192 * 1024>>>(g, rnd, (int)hr.size(), iters, half, out);
      report_pipe("pipe x3");
    }
  }
  // sensitivity of the copy rate to the instructions spent per copy (7 warps, 40 MB, 3 stages)
  cudaFuncSetAttribute(gather_pipe<3, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
  cudaFuncSetAttribute(gather_pipe<3, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
  {
    const size_t half = (40ull << 20) / 2;
    auto rep_x = [&](int extra) {
      cudaDeviceSynchronize();
      std::vector<long long> h(148);
      cudaMemcpy(h.data(), out, 148 * 8, cudaMemcpyDeviceToHost);
      double avg = 0;
      for (auto v : h) avg += (double)v;
      avg /= 148;
      printf("footprint 40 MB  7 warps pipe x3 +%d int ops/copy %7.0f cycles/64KB stage  %5.1f B/cycle/SM\n", extra,
             avg / iters, 65536.0 * iters / avg);
    };
    for (int rep = 0; rep < 2; ++rep)
      gather_pipe<3, 0><<<148, 224, 192 * 1024>>>(g, rnd, (int)hr.size(), iters, half, out, 0u);
    rep_x(0);
    for (int rep = 0; rep < 2; ++rep)
      gather_pipe<3, 4><<<148, 224, 192 * 1024>>>(g, rnd, (int)hr.size(), iters, half, out, 0u);
    rep_x(4);
    for (int rep = 0; rep < 2; ++rep)
      gather_pipe<3, 8><<<148, 224, 192 * 1024>>>(g, rnd, (int)hr.size(), iters, half, out, 0u);
    rep_x(8);
  }
  int herr = 0;
  cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
  printf("bulk wait timeouts: %d; status: %s\n", herr, cudaGetErrorString(cudaGetLastError()));
  return herr != 0;
}
