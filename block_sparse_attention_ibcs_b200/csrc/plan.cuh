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
// fits, otherwise re-read from global memory (L2) on each pass.  Passes over the row:
// staging with the positive count and sum; a water-filling estimate of lambda (usually
// one pass); F at the estimate and at one Newton step from it (these bracket lambda* to
// one ulp on typical rows; otherwise a doubling search and bisection follow); the codes
// (q_j or "saturated") with per-thread sums; and the output pass.  The number selected
// in each thread's contiguous chunk needs no pass of its own: non-saturated intervals are
// shorter than 2^32, so the chunk's blocks hold exactly the lattice points of the chunk's
// (contiguous) interval.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_SMEM_MAX_FLOATS = 40 * 1024;  // 160 KB of staged row
constexpr uint64_t TWO32 = 1ull << 32;

struct PlanArgs {
  const float* S;   // [rows, nK] (not read in the uniform variant)
  int32_t* idx;     // [rows, s]
  float* logpi;     // [rows, s]
  int nK, s;
  uint64_t seed, offset;
  int mode;         // ab_plan_mode: SIP, SIP without inverse-probability weights, uniform
  int row0;         // row index of this launch's first row in the whole (b, h, i) order
                    // (the Philox counter uses it: a launch over a slice of heads draws as
                    // the full launch would)
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

// q_j(lambda) = floor(fl32(lambda * S_j) * 2^32) for fl32(lambda S_j) < 1, exactly, from
// the fp32 bit pattern: x = m 2^(e-150) with the 24-bit significand m, so x 2^32 =
// (m 2^8) >> (126 - e); (b << 8) | 2^31 is m 2^8, and the clamping funnel shift turns
// shifts of 32 or more into 0 (x < 2^-32 or zero; a negative or NaN x wraps to such a
// shift too, so scores that are not positive contribute 0).  Returns whether x >= 1, where
// q_j = 2^32 instead.  __fmul_rn keeps the product a single fp32 rounding.
AB_DEV bool fixed_q32(float lam, float sv, uint32_t& q) {
  const float x = __fmul_rn(lam, sv);
  const uint32_t b = __float_as_uint(x);
  q = __funnelshift_rc((b << 8) | 0x80000000u, 0u, 126u - (b >> 23));
  return x >= 1.0f;
}

// F's per-thread part: saturated blocks add 2^32, the others q_j.
AB_DEV void add_q(float lam, float sv, uint64_t& acc) {
  uint32_t q;
  const bool sat = fixed_q32(lam, sv, q);
  acc += sat ? TWO32 : (uint64_t)q;
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

// Exclusive block scans of two uint64 values in thread order, one pair of barriers;
// returns this thread's prefixes and the block totals.
AB_DEV void block_exscan2_u64(uint64_t v0, uint64_t v1, uint64_t* red0, uint64_t* red1,
                              uint64_t& before0, uint64_t& before1, uint64_t& total0,
                              uint64_t& total1) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  uint64_t inc0 = v0, inc1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y0 = __shfl_up_sync(0xffffffffu, inc0, o);
    const uint64_t y1 = __shfl_up_sync(0xffffffffu, inc1, o);
    if (l >= o) {
      inc0 += y0;
      inc1 += y1;
    }
  }
  __syncthreads();
  if (l == 31) {
    red0[w] = inc0;
    red1[w] = inc1;
  }
  __syncthreads();
  uint64_t b0 = 0, b1 = 0, t0 = 0, t1 = 0;
#pragma unroll
  for (int i = 0; i < PLAN_WARPS; ++i) {
    if (i < w) {
      b0 += red0[i];
      b1 += red1[i];
    }
    t0 += red0[i];
    t1 += red1[i];
  }
  before0 = b0 + inc0 - v0;
  before1 = b1 + inc1 - v1;
  total0 = t0;
  total1 = t1;
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
  const bool uniform = a.mode == AB_PLAN_UNIFORM;
  // score j of the row when it is not staged (the uniform variant reads no scores)
  auto sv_at = [&](int j) -> float { return uniform ? 1.f : __ldg(grow + j); };
  const int nK4 = (nK + 3) >> 2;  // staged row padded with zeros to whole float4s
  const uint64_t s = (uint64_t)a.s;
  const uint64_t target = s * TWO32;

  // ---- positive blocks and their total score (fewer than s positive blocks = budget
  // unreachable); per-thread sums in compensated fp32, block sum in fp64.  With the row
  // staged in shared memory this pass also copies it there.
  uint64_t npos = 0;
  double tot = 0.0;
  {
    float sum = 0.f, comp = 0.f;
    auto acc = [&](float sv) {
      if (sv > 0.f) {
        const float y = sv - comp, t2 = sum + y;
        comp = (t2 - sum) - y;
        sum = t2;
        ++npos;
      }
    };
    if (STAGED) {
      const bool vec = ((uintptr_t)grow & 15u) == 0 && (nK & 3) == 0;
      float4* s4 = reinterpret_cast<float4*>(srow_smem);
      for (int j = tid; j < nK4; j += PLAN_THREADS) {
        float4 v;
        if (uniform) {  // the same score for every block
          v.x = (4 * j < nK) ? 1.f : 0.f;
          v.y = (4 * j + 1 < nK) ? 1.f : 0.f;
          v.z = (4 * j + 2 < nK) ? 1.f : 0.f;
          v.w = (4 * j + 3 < nK) ? 1.f : 0.f;
        } else if (vec) {
          v = __ldg(reinterpret_cast<const float4*>(grow) + j);
        } else {
          v.x = (4 * j < nK) ? __ldg(grow + 4 * j) : 0.f;
          v.y = (4 * j + 1 < nK) ? __ldg(grow + 4 * j + 1) : 0.f;
          v.z = (4 * j + 2 < nK) ? __ldg(grow + 4 * j + 2) : 0.f;
          v.w = (4 * j + 3 < nK) ? __ldg(grow + 4 * j + 3) : 0.f;
        }
        s4[j] = v;
        acc(v.x);
        acc(v.y);
        acc(v.z);
        acc(v.w);
      }
      srow = srow_smem;  // read only after the barriers of the block sum below
    } else {
      for (int j = tid; j < nK; j += PLAN_THREADS) acc(sv_at(j));
    }
    tot = (double)sum - (double)comp;
  }
  block_sum_cd(npos, tot, red, redd);
  const bool reachable = npos >= s;

  // ---- lambda*: the smallest positive fp32 (bit pattern in (0, 0x7F800000]) with
  // F(lambda) >= s 2^32.  F is monotone in the bit pattern, so any search that brackets
  // the boundary and bisects finds the same lambda as a full 31-step bisection.
  auto F = [&](uint32_t bits) -> uint64_t {
    const float lam = __uint_as_float(bits);
    uint64_t part = 0;
    if (STAGED) {
      const float4* s4 = reinterpret_cast<const float4*>(srow);
      for (int j = tid; j < nK4; j += PLAN_THREADS) {
        const float4 v = s4[j];
        add_q(lam, v.x, part);
        add_q(lam, v.y, part);
        add_q(lam, v.z, part);
        add_q(lam, v.w, part);
      }
    } else {
      for (int j = tid; j < nK; j += PLAN_THREADS) add_q(lam, sv_at(j), part);
    }
    return block_sum_u64(part, red);
  };
  uint32_t lo = 0u, hi = 0x7F800000u;
  if (reachable) {
    // Water filling in fp64 (a starting point only): lambda <- (s - |saturated|) / (sum of
    // the unsaturated scores) until the saturated set stops growing; in practice one or
    // two rounds, ending within an ulp or two of lambda*.
    double lam_w = (tot > 0.0) ? (double)a.s / tot : 0.0;
    double rest_est = tot;
    for (int it = 0; it < 32 && lam_w > 0.0; ++it) {
      uint64_t nsat = 0;
      double rest = 0.0;
      const float lw = (float)lam_w;
      {
        float sum = 0.f, comp = 0.f;
        for (int j = tid; j < nK; j += PLAN_THREADS) {
          const float sv = STAGED ? srow[j] : sv_at(j);
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
  // positive block is SAT and the others have code 0).  With the row staged in shared
  // memory the codes overwrite the thread's own slots: every read of the scores by the
  // other threads happened before the barriers of the last block sum.
  constexpr uint32_t SAT = 0xFFFFFFFFu;
  uint32_t* code_smem = reinterpret_cast<uint32_t*>(srow_smem);
  auto code_from_score = [&](float sv) -> uint32_t {
    if (reachable) {
      uint32_t q;
      return fixed_q32(lam, sv, q) ? SAT : q;
    }
    return (sv > 0.f) ? SAT : 0u;
  };
  const int per = (nK + PLAN_THREADS - 1) / PLAN_THREADS;
  const int j0 = min(nK, tid * per), j1 = min(nK, j0 + per);
  // my_rest: the chunk's total q (budget reachable) or its number of code-0 blocks
  uint64_t my_sat = 0, my_rest = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t c = code_from_score(STAGED ? srow[j] : sv_at(j));
    if (STAGED) code_smem[j] = c;
    if (c == SAT) ++my_sat;
    else my_rest += reachable ? c : 1u;
  }
  uint64_t sat_before, rest_before, n_sat, tot_rest;
  block_exscan2_u64(my_sat, my_rest, red, red2, sat_before, rest_before, n_sat, tot_rest);

  const uint32_t U = philox4x32_10_w0((uint32_t)(a.row0 + row), (uint32_t)a.offset, (uint32_t)(a.offset >> 32),
                                      0u, (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
  // lattice points U + k 2^32 below x, for 0 <= x <= s 2^32 (U < 2^32)
  const uint64_t CB = TWO32 - 1u - (uint64_t)U;
  auto below = [&](uint64_t x) -> uint64_t { return (x + CB) >> 32; };
  // Saturated blocks come first in the layout, block k of them covering [k 2^32, (k+1) 2^32):
  // each holds exactly one lattice point, so every saturated block is drawn.  The other
  // blocks follow in ascending order; this thread's chunk covers [start, start + my_rest).
  // With the budget unreachable, the first s - n_sat code-0 blocks (in order) complete it.
  const uint64_t start = n_sat * TWO32 + rest_before;
  const uint64_t need = s - min(n_sat, s);
  const uint64_t my_sel =
      my_sat + (reachable ? below(min(start + my_rest, target)) - below(min(start, target))
                          : (rest_before < need ? min(my_rest, need - rest_before) : 0ull));
  uint64_t out_before, zero_b, n_sel, zero_t;
  block_exscan2_u64(my_sel, 0ull, red, red2, out_before, zero_b, n_sel, zero_t);
  if (n_sel != s && tid == 0) ab_flag(AB_ERR_DEVICE_CHECK);  // cannot happen; guards the writes

  // ---- write ascending idx and the fixed-point probability (its log follows below)
  {
    uint64_t pos = start, zero_i = rest_before;
    uint64_t o = out_before;
    int32_t* oidx = a.idx + (size_t)row * a.s;
    uint32_t* oraw = reinterpret_cast<uint32_t*>(a.logpi + (size_t)row * a.s);
    for (int j = j0; j < j1; ++j) {
      const uint32_t c = STAGED ? code_smem[j] : code_from_score(sv_at(j));
      bool sel;
      uint32_t qq = 0xFFFFFFFFu;  // pi = 1 (a capped or ordinary q is at most 2^32 - 256)
      if (c == SAT) {
        sel = true;
      } else if (reachable) {
        const uint64_t st = min(pos, target), en = min(pos + c, target);
        sel = below(en) != below(st);
        qq = (uint32_t)(en - st);
        pos += c;
      } else {
        sel = zero_i++ < need;
      }
      if (sel) {
        if (o < s) {
          oidx[o] = j;
          oraw[o] = qq;
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
      olp[o] = (q == 0xFFFFFFFFu || a.mode == AB_PLAN_SIP_NO_IPW)
                   ? 0.f
                   : (float)log((double)q * (1.0 / 4294967296.0));
    }
  }
}

// ---------------------------------------------------------------------------- top-k
//
// Top-k variant of the planner (AB-Attention page, ablations: the deterministic top-k
// selection SIP is compared against): per row, the s blocks with the largest scores, ties
// to the lower block index, ascending; log pi = 0 (pi = 1 for every kept block, no
// reweighting).  Scores are ranked by an order-preserving 32-bit key (score_key: larger
// score, larger key; +0 above -0; NaN below every number).  A 4-pass radix select (8-bit
// digits from the top) finds the key K* of the s-th largest; every key > K* is kept, plus
// the first s - |{key > K*}| keys equal to K* in block order.

AB_DEV uint32_t score_key(float v) {
  const uint32_t b = __float_as_uint(v);
  if (v != v) return 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <bool STAGED>
__global__ void __launch_bounds__(PLAN_THREADS) topk_kernel(PlanArgs a) {
  extern __shared__ uint32_t key_smem[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel_digit, sel_above;
  __shared__ uint64_t red[PLAN_WARPS];
  __shared__ uint64_t red2[PLAN_WARPS];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nK = a.nK;
  const float* grow = a.S + (size_t)row * nK;
  auto key_at = [&](int j) -> uint32_t { return STAGED ? key_smem[j] : score_key(__ldg(grow + j)); };
  if (STAGED) {
    for (int j = tid; j < nK; j += PLAN_THREADS) key_smem[j] = score_key(__ldg(grow + j));
  }
  uint32_t prefix = 0u, mask = 0u;
  uint32_t remaining = (uint32_t)a.s;  // rank of K* among the keys matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += PLAN_THREADS) hist[b] = 0u;
    __syncthreads();  // also orders the staging above before the first histogram
    for (int j = tid; j < nK; j += PLAN_THREADS) {
      const uint32_t k = key_at(j);
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits 255 - 8l down to 248 - 8l; find the digit where the count of
      // keys at or above it first reaches `remaining`
      uint32_t own = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) own += hist[255 - 8 * tid - i];
      uint32_t inc = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (tid >= o) inc += y;
      }
      const uint32_t before = inc - own;  // keys in higher digits of the lanes before
      const bool mine = before < remaining && inc >= remaining;
      if (mine) {
        uint32_t above = before;
        for (int i = 0; i < 8; ++i) {
          const uint32_t dgt = 255u - 8u * tid - i;
          const uint32_t c = hist[dgt];
          if (above + c >= remaining) {
            sel_digit = dgt;
            sel_above = above;
            break;
          }
          above += c;
        }
      }
    }
    __syncthreads();
    prefix |= sel_digit << shift;
    mask |= 255u << shift;
    remaining -= sel_above;
    __syncthreads();  // sel_digit / sel_above are rewritten by the next pass
  }
  const uint32_t kstar = prefix;
  const uint64_t need_eq = remaining;  // keys equal to K* to keep (>= 1)

  // keep every key > K* and the first need_eq keys == K*; contiguous chunks keep block order
  const int per = (nK + PLAN_THREADS - 1) / PLAN_THREADS;
  const int j0 = min(nK, tid * per), j1 = min(nK, j0 + per);
  uint64_t my_gt = 0, my_eq = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t k = key_at(j);
    my_gt += k > kstar;
    my_eq += k == kstar;
  }
  uint64_t gt_before, eq_before, n_gt, n_eq;
  block_exscan2_u64(my_gt, my_eq, red, red2, gt_before, eq_before, n_gt, n_eq);
  const uint64_t my_sel = my_gt + (eq_before < need_eq ? min(my_eq, need_eq - eq_before) : 0ull);
  uint64_t out_before, zb, n_sel, zt;
  block_exscan2_u64(my_sel, 0ull, red, red2, out_before, zb, n_sel, zt);
  if (n_sel != (uint64_t)a.s && tid == 0) ab_flag(AB_ERR_DEVICE_CHECK);  // cannot happen
  uint64_t o = out_before, eq_i = eq_before;
  int32_t* oidx = a.idx + (size_t)row * a.s;
  float* olp = a.logpi + (size_t)row * a.s;
  for (int j = j0; j < j1; ++j) {
    const uint32_t k = key_at(j);
    const bool sel = k > kstar || (k == kstar && eq_i++ < need_eq);
    if (sel) {
      if (o < (uint64_t)a.s) {
        oidx[o] = j;
        olp[o] = 0.f;
      }
      ++o;
    }
  }
}

}  // namespace abattn
