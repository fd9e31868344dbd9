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

// floor(x * 2^32) for 0 <= x < 1, exactly, from the fp32 bit pattern: x = m 2^(e-150) with
// the 24-bit significand m, so x 2^32 = m 2^(e-118) (at most 2^32 - 2^8: fits 32 bits).
AB_DEV uint32_t frac32(float x) {
  const uint32_t b = __float_as_uint(x);
  const int e = (int)(b >> 23);
  const uint32_t m = (b & 0x7FFFFFu) | 0x800000u;
  if (e >= 118) return m << (e - 118);
  const int sh = 118 - e;
  return sh < 32 ? (m >> sh) : 0u;  // also 0 for zero and subnormal x (far below 2^-32)
}

// q_j(lambda) in 2^-32 units.  __fmul_rn keeps the product a single fp32 rounding.
AB_DEV uint64_t fixed_q(float lam, float sv) {
  if (!(sv > 0.f)) return 0ull;
  const float x = __fmul_rn(lam, sv);
  if (x >= 1.0f) return TWO32;
  return (uint64_t)frac32(x);
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

// Block-wide sums of a (uint64 count, fp64 value) pair, one pair of barriers.
AB_DEV void block_sum_cd(uint64_t& c, double& v, uint64_t* redc, double* redv) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    v += __shfl_xor_sync(0xffffffffu, v, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) { redc[w] = c; redv[w] = v; }
  __syncthreads();
  c = 0;
  v = 0.0;
#pragma unroll
  for (int i = 0; i < PLAN_WARPS; ++i) { c += redc[i]; v += redv[i]; }
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
  __shared__ double redd[PLAN_WARPS];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nK = a.nK;
  const float* grow = a.S + (size_t)row * nK;
  const float* srow = grow;
  const int nK4 = (nK + 3) >> 2;  // staged row padded with zeros to whole float4s
  if (STAGED) {
    for (int j = tid; j < nK4 * 4; j += PLAN_THREADS) srow_smem[j] = (j < nK) ? __ldg(grow + j) : 0.f;
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
    if (STAGED) {
      const float4* s4 = reinterpret_cast<const float4*>(srow);
      for (int j = tid; j < nK4; j += PLAN_THREADS) {
        const float4 v = s4[j];
        part += fixed_q(lam, v.x) + fixed_q(lam, v.y) + fixed_q(lam, v.z) + fixed_q(lam, v.w);
      }
    } else {
      for (int j = tid; j < nK; j += PLAN_THREADS) part += fixed_q(lam, srow[j]);
    }
    return block_sum_u64(part, red);
  };
  uint32_t lo = 0u, hi = 0x7F800000u;
  // positive blocks and their total score; fewer than s positive blocks = budget unreachable
  // per-thread sums in compensated fp32 (no per-element fp64 conversions), block sum in fp64
  uint64_t npos = 0;
  double tot = 0.0;
  {
    float sum = 0.f, comp = 0.f;
    for (int j = tid; j < nK; j += PLAN_THREADS) {
      const float sv = srow[j];
      if (sv > 0.f) {
        const float y = sv - comp, t2 = sum + y;
        comp = (t2 - sum) - y;
        sum = t2;
        ++npos;
      }
    }
    tot = (double)sum - (double)comp;
  }
  block_sum_cd(npos, tot, red, redd);
  const bool reachable = npos >= s;
  if (reachable) {
    // Water filling in fp64 (a starting point only): lambda <- (s - |saturated|) / (sum of
    // the unsaturated scores) until the saturated set stops growing; in practice a few
    // rounds, ending within an ulp or two of lambda*.
    double lam_w = (tot > 0.0) ? (double)a.s / tot : 0.0;
    double rest_est = tot;
    for (int it = 0; it < 32 && lam_w > 0.0; ++it) {
      uint64_t nsat = 0;
      double rest = 0.0;
      const float lw = (float)lam_w;
      {
        float sum = 0.f, comp = 0.f;
        for (int j = tid; j < nK; j += PLAN_THREADS) {
          const float sv = srow[j];
          if (sv > 0.f) {
            if (__fmul_rn(lw, sv) >= 1.f) {
              ++nsat;
            } else {
              const float y = sv - comp, t2 = sum + y;
              comp = (t2 - sum) - y;
              sum = t2;
            }
          }
        }
        rest = (double)sum - (double)comp;
      }
      block_sum_cd(nsat, rest, red, redd);
      rest_est = rest;
      if (nsat >= (uint64_t)a.s || !(rest > 0.0)) break;
      const double nxt = (double)((uint64_t)a.s - nsat) / rest;
      if (!(nxt > lam_w)) break;  // converged (the iteration only increases)
      lam_w = nxt;
    }
    const float lam_est = (float)lam_w;
    uint32_t b = __float_as_uint(lam_est);
    if (!(lam_est > 0.f) || !isfinite(lam_est)) b = 0x3F800000u;  // 1.0: any start works
    uint64_t fb = F(b);
    // one Newton step on the fixed-point sum: F grows by about rest * 2^32 per unit lambda
    if (rest_est > 0.0 && isfinite(lam_est) && lam_est > 0.f) {
      const double lam_n = (double)__uint_as_float(b) +
                           ((double)target - (double)fb) / (rest_est * 4294967296.0);
      const float lf = (float)lam_n;
      if (lf > 0.f && isfinite(lf) && __float_as_uint(lf) != b) {
        const uint32_t b2 = __float_as_uint(lf);
        const uint64_t f2 = F(b2);
        // keep whichever point is on the same side as the boundary search needs
        if ((f2 >= target) == (fb >= target)) { b = b2; fb = f2; }
        else if (b2 > b) { lo = b; hi = b2; }
        else { lo = b2; hi = b; }
      }
    }
    const bool bracketed = !(lo == 0u && hi == 0x7F800000u);  // by the Newton point
    if (!bracketed) {
      if (fb >= target) {  // boundary at or below b: step down
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
          // the probability's fixed-point value for now (2^32 - 1 stands for pi = 1: a capped
          // or ordinary q is at most 2^32 - 256); its log follows in a compacted pass
          reinterpret_cast<uint32_t*>(olp)[o] = (qq == TWO32) ? 0xFFFFFFFFu : (uint32_t)qq;
        }
        ++o;
      }
    }
  }
  // log(pi) for the s outputs, spread evenly over the threads (no divergent fp64 log)
  __syncthreads();
  {
    float* olp = a.logpi + (size_t)row * a.s;
    uint32_t* raw = reinterpret_cast<uint32_t*>(olp);
    for (int o = tid; o < a.s; o += PLAN_THREADS) {
      const uint32_t q = raw[o];
      olp[o] = (q == 0xFFFFFFFFu) ? 0.f : (float)log((double)q * (1.0 / 4294967296.0));
    }
  }
}

}  // namespace abattn
