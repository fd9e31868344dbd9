// SIP planner for sm_100a: inclusion probabilities and systematic sampling.
//
// AB-Attention page (onedev.kr/papers/1521), section "how to use": each query block
// turns its block scores S_j into inclusion probabilities pi_j = min(1, lambda S_j)
// with sum_j pi_j = s, keeps every pi = 1 block, and draws exactly s distinct blocks
// by systematic sampling; all queries of the block share the draw.
//
// Arithmetic (identical on every device and on the CPU, so plans are bit-exact):
//   x_j = fl32(lambda * S_j) (one rounding, never fused), q_j = 2^32 if x_j >= 1 else
//   floor(x_j * 2^32); F(lambda) = sum q_j in uint64 (order-free).  lambda* = the
//   smallest positive fp32 with F >= s * 2^32, found by bisection over fp32 bit patterns.
//   Layout: saturated blocks first (ascending j, each exactly 2^32 long), then the rest
//   (ascending j); positions are capped at s * 2^32, which trims only the tail of the
//   non-saturated blocks.  Block j is sampled iff a lattice point U + k 2^32 falls in
//   its interval, with U = word 0 of Philox4x32-10(key = seed, counter = (row, offset_lo,
//   offset_hi, 0)).
//
// One CTA of PLAN_THREADS threads per row.  The row is staged in shared memory when it
// fits, otherwise re-read from global memory (L2) on each bisection step.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_SMEM_MAX_FLOATS = 40 * 1024;  // 160 KB of staged row
constexpr uint64_t TWO32 = 1ull << 32;

struct PlanArgs {
  const float* S;   // [rows, nK]
  int32_t* idx;     // [rows, s]
  float* logpi;     // [rows, s]
  int nK, s;
  uint64_t seed, offset;
};

// Philox4x32-10 (Salmon et al., SC'11), word 0 of the output block.
AB_DEV uint32_t philox4x32_10_w0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                 uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

// q_j(lambda) in 2^-32 units.  __fmul_rn keeps the product a single fp32 rounding.
AB_DEV uint64_t fixed_q(float lam, float sv) {
  if (!(sv > 0.f)) return 0ull;
  const float x = __fmul_rn(lam, sv);
  if (x >= 1.0f) return TWO32;
  return (uint64_t)__float2ull_rz(__fmul_rn(x, 4294967296.0f));  // exact scaling, truncation
}

// Block-wide sum of a uint64 (all threads get the result).  red: PLAN_WARPS slots.
AB_DEV uint64_t block_sum_u64(uint64_t v, uint64_t* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  uint64_t tot = 0;
#pragma unroll
  for (int i = 0; i < PLAN_WARPS; ++i) tot += red[i];
  return tot;
}

// Block-wide fp32 sum (all threads get the result).
AB_DEV float block_sum_f32(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < PLAN_WARPS; ++i) tot += red[i];
  return tot;
}

// Exclusive block scan of uint64 values in thread order; returns this thread's prefix.
AB_DEV uint64_t block_exscan_u64(uint64_t v, uint64_t* red, uint64_t* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  uint64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (l >= o) inc += y;
  }
  __syncthreads();
  if (l == 31) red[w] = inc;
  __syncthreads();
  uint64_t before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < PLAN_WARPS; ++i) {
    if (i < w) before += red[i];
    tot += red[i];
  }
  *total = tot;
  return before + inc - v;
}

template <bool STAGED>
__global__ void __launch_bounds__(PLAN_THREADS) plan_kernel(PlanArgs a) {
  extern __shared__ float srow_smem[];
  __shared__ uint64_t red[PLAN_WARPS];
  __shared__ uint64_t red2[PLAN_WARPS];
  __shared__ float redf[PLAN_WARPS];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nK = a.nK;
  const float* grow = a.S + (size_t)row * nK;
  const float* srow = grow;
  if (STAGED) {
    for (int j = tid; j < nK; j += PLAN_THREADS) srow_smem[j] = __ldg(grow + j);
    __syncthreads();
    srow = srow_smem;
  }
  const uint64_t s = (uint64_t)a.s;
  const uint64_t target = s * TWO32;

  // ---- lambda*: the smallest positive fp32 (bit pattern in (0, 0x7F800000]) with
  // F(lambda) >= s 2^32.  F is monotone in the bit pattern, so any search that brackets
  // the boundary and bisects finds the same lambda as a full 31-step bisection.  A
  // water-filling estimate lambda <- (s - |saturated|) / (sum of the unsaturated S)
  // starts the search a few ulps from the boundary.
  auto F = [&](uint32_t bits) -> uint64_t {
    const float lam = __uint_as_float(bits);
    uint64_t part = 0;
    for (int j = tid; j < nK; j += PLAN_THREADS) part += fixed_q(lam, srow[j]);
    return block_sum_u64(part, red);
  };
  uint32_t lo = 0u, hi = 0x7F800000u;
  const bool reachable = F(hi) >= target;
  if (reachable) {
    // water-filling estimate in fp32 (only a starting point)
    float lam_est = 0.f;
    {
      float part = 0.f;
      for (int j = tid; j < nK; j += PLAN_THREADS) part += fmaxf(srow[j], 0.f);
      float tot = block_sum_f32(part, redf);
      lam_est = (tot > 0.f) ? (float)a.s / tot : 0.f;
      for (int it = 0; it < 8 && lam_est > 0.f && isfinite(lam_est); ++it) {
        float rest = 0.f;
        uint32_t nsat = 0;
        for (int j = tid; j < nK; j += PLAN_THREADS) {
          const float sv = srow[j];
          if (sv > 0.f) {
            if (__fmul_rn(lam_est, sv) >= 1.f) ++nsat; else rest += sv;
          }
        }
        const uint64_t ns = block_sum_u64(nsat, red);
        rest = block_sum_f32(rest, redf);
        if (ns >= (uint64_t)a.s || !(rest > 0.f)) break;
        const float nxt = (float)((uint64_t)a.s - ns) / rest;
        if (!(nxt > lam_est)) break;  // converged (the iteration only increases)
        lam_est = nxt;
      }
    }
    uint32_t b = __float_as_uint(lam_est);
    if (!(lam_est > 0.f) || !isfinite(lam_est)) b = 0x3F800000u;  // 1.0: any start works
    if (F(b) >= target) {  // boundary at or below b: step down
      hi = b;
      uint32_t step = 1;
      while (true) {
        const uint32_t cand = (hi > step) ? hi - step : 0u;
        if (cand == 0u || F(cand) < target) { lo = cand; break; }
        hi = cand;
        step <<= 1;
      }
    } else {  // boundary above b: step up
      lo = b;
      uint32_t step = 1;
      while (true) {
        const uint32_t cand = (0x7F800000u - lo > step) ? lo + step : 0x7F800000u;
        if (cand == 0x7F800000u || F(cand) >= target) { hi = cand; break; }
        lo = cand;
        step <<= 1;
      }
    }
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      if (F(mid) >= target) hi = mid; else lo = mid;
    }
  }
  const float lam = __uint_as_float(hi);

  // ---- per element code on this thread's contiguous chunk: the fixed-point q_j (< 2^32 - 255)
  // or SAT for an inclusion probability of exactly 1 (when the budget is unreachable: every
  // positive block is SAT and zero blocks have code 0).  With the row staged in shared
  // memory the codes overwrite the thread's own slots, so the two selection passes below
  // are integer-only.
  constexpr uint32_t SAT = 0xFFFFFFFFu;
  uint32_t* code_smem = reinterpret_cast<uint32_t*>(srow_smem);
  auto code_from_score = [&](float sv) -> uint32_t {
    if (reachable) {
      const uint64_t q = fixed_q(lam, sv);
      return q == TWO32 ? SAT : (uint32_t)q;
    }
    return (sv > 0.f) ? SAT : 0u;
  };
  auto code_of = [&](int j) -> uint32_t {
    if (STAGED) return code_smem[j];
    return code_from_score(srow[j]);
  };
  const int per = (nK + PLAN_THREADS - 1) / PLAN_THREADS;
  const int j0 = min(nK, tid * per), j1 = min(nK, j0 + per);
  uint64_t my_sat = 0, my_rest = 0, my_zero = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t c = code_from_score(srow[j]);
    if (STAGED) code_smem[j] = c;  // own slot; every read of the scores happened before
    if (c == SAT) ++my_sat;
    else if (reachable) my_rest += c;
    else ++my_zero;
  }
  uint64_t n_sat = 0, tot_rest = 0, n_zero_tot = 0;
  const uint64_t sat_before = block_exscan_u64(my_sat, red, &n_sat);
  const uint64_t rest_before = block_exscan_u64(my_rest, red2, &tot_rest);
  uint64_t zero_before = 0;
  if (!reachable) zero_before = block_exscan_u64(my_zero, red, &n_zero_tot);

  const uint32_t U = philox4x32_10_w0((uint32_t)row, (uint32_t)a.offset, (uint32_t)(a.offset >> 32),
                                      0u, (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
  // lattice points U + k 2^32 below x (x <= s 2^32, so at most s)
  auto below = [&](uint64_t x) -> uint64_t { return x > U ? ((x - U - 1) >> 32) + 1 : 0ull; };
  // Saturated blocks come first in the layout, block k of them covering [k 2^32, (k+1) 2^32):
  // each holds exactly one lattice point, so every saturated block is drawn.

  // ---- selection flags, counted per chunk
  uint64_t my_sel = 0;
  {
    uint64_t pos = n_sat * TWO32 + rest_before, zero_i = zero_before;
    for (int j = j0; j < j1; ++j) {
      const uint32_t c = code_of(j);
      bool sel;
      if (c == SAT) {
        sel = true;
      } else if (reachable) {
        const uint64_t st = min(pos, target), en = min(pos + c, target);
        sel = below(en) > below(st);
        pos += c;
      } else {
        sel = zero_i++ < s - n_sat;
      }
      my_sel += sel;
    }
  }
  uint64_t n_sel = 0;
  const uint64_t out_before = block_exscan_u64(my_sel, red, &n_sel);
  if (n_sel != s && tid == 0) ab_flag(AB_ERR_DEVICE_CHECK);  // cannot happen; guards the writes

  // ---- write ascending idx and log(pi)
  {
    uint64_t pos = n_sat * TWO32 + rest_before, zero_i = zero_before;
    uint64_t o = out_before;
    int32_t* oidx = a.idx + (size_t)row * a.s;
    float* olp = a.logpi + (size_t)row * a.s;
    for (int j = j0; j < j1; ++j) {
      const uint32_t c = code_of(j);
      bool sel;
      uint64_t qq = TWO32;
      if (c == SAT) {
        sel = true;
      } else if (reachable) {
        const uint64_t st = min(pos, target), en = min(pos + c, target);
        sel = below(en) > below(st);
        qq = en - st;
        pos += c;
      } else {
        sel = zero_i++ < s - n_sat;
      }
      if (sel) {
        if (o < s) {
          oidx[o] = j;
          olp[o] = (qq == TWO32) ? 0.f : (float)log((double)qq * (1.0 / 4294967296.0));
        }
        ++o;
      }
    }
  }
}

}  // namespace abattn
