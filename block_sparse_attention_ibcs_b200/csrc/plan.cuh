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
// One CTA of PLAN_THREADS threads per row, three per SM.  The row's first
// PLAN_STAGE_FLOAT4S float4s (all of a Wan-sized row) are staged in shared memory by one
// bulk copy; the rest of a longer row is re-read from global memory (L2) on each pass.  Passes over
// the row: staging with the positive count and sum; F at the three fp32 neighbours of
// lambda0 = s / sum(S) (with the sum of the scores unsaturated at lambda0) -- without
// saturation lambda* is lambda0 or its upper neighbour, so this one pass brackets it --
// then, for the rows it does not bracket, a Newton step, doubling steps and bisection;
// and the output pass.  After staging every pass walks the thread's contiguous chunk, so
// the evaluation at lambda* already gives each thread its saturated count and q sum; the
// number drawn before a chunk needs no pass: non-saturated intervals are shorter than
// 2^32, so the blocks before it hold exactly the lattice points of their (contiguous)
// interval.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_SMEM_MAX_FLOATS = 40 * 1024;  // 160 KB of staged row (top-k keys)
// The SIP planner stages at most the first PLAN_STAGE_FLOAT4S float4s of a row (75,760
// bytes) in shared memory, so that three rows fit on an SM (228 KB, less the 1,040 bytes of
// static shared memory and the 1 KB the system reserves per block); a longer row reads its
// tail from global memory.  Measured on B200: three rows per SM instead of two took the
// Wan2.1-14B planner (18,900 blocks, fully staged) from 1.90 to 1.64 ms.
constexpr int PLAN_STAGE_FLOAT4S = 4735;
constexpr uint64_t TWO32 = 1ull << 32;
constexpr uint64_t kPlanTimeoutNs = 2000000000ull;  // bounded wait for the staged row

struct PlanArgs {
  const float* S;   // [rows, nK] (not read in the uniform variant)
  int32_t* idx;     // [rows, s]
  float* logpi;     // [rows, s]
  int nK, s;
  uint64_t seed, offset;
  int mode;         // ab_plan_mode: SIP, SIP without inverse-probability weights, uniform
  // Philox row numbering.  Launch row r is query block r % nQ of (b, h) = the flattened
  // head bh0 + r / nQ of the call (B x H heads); the draw uses that row's index in the
  // whole layer, (b * Ht + h0 + h) * nQ + i, so a launch over a slice of the call, or a
  // call over a slice of a layer's heads, draws exactly as one launch over the layer.
  int nQ, H, Ht, h0;
  long long bh0;
};

// Counter word of launch row r (fits 32 bits: the host checks B * Ht * nQ < 2^31).
AB_DEV uint32_t plan_counter_row(const PlanArgs& a, int r) {
  const long long bl = a.bh0 + r / a.nQ;
  const int i = r - (r / a.nQ) * a.nQ;
  const long long b = bl / a.H, h = bl - b * a.H;
  return (uint32_t)((b * a.Ht + a.h0 + h) * a.nQ + i);
}

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

// The same step in a form that runs mostly on the FMA pipe, for lambda < 2^95 (every row
// but pathological ones).  With L = lambda 2^32 (an exact scaling), y = fl(L S_j) equals
// fl(lambda S_j) 2^32 exactly while lambda S_j lies in fp32's normal range, and below it
// both floors are 0.  cvt.rzi.u32 of y is floor(y) = q_j for y < 2^32 (the largest fp32
// below 2^32 is 2^32 - 256), saturates to 2^32 - 1 for y >= 2^32 (lambda S_j >= 1), and
// gives 0 for a negative or NaN y.  So over a set of blocks F = sum cvt(y_j) + n_sat, and
// the saturation test y >= 2^32 is sat(y - (2^32 - 256)), exactly 0 or 1 (NaN: 0).
constexpr float LAM_FAST_MAX = 39614081257132168796771975168.f;  // 2^95
constexpr float TWO32F = 4294967296.f;
constexpr float BELOW_TWO32F = 4294967040.f;

AB_DEV uint32_t f2u_rz(float y) {
  uint32_t q;
  asm("cvt.rzi.u32.f32 %0, %1;" : "=r"(q) : "f"(y));
  return q;
}
// 1 if y >= 2^32, else 0 (y an fp32 product as above)
AB_DEV float sat_flag(float y) {
  float t;
  asm("add.rn.sat.f32 %0, %1, %2;" : "=f"(t) : "f"(y), "f"(-BELOW_TWO32F));
  return t;
}
// acc + q as one wide multiply-add
AB_DEV uint64_t add_wide(uint64_t acc, uint32_t q) {
  uint64_t r;
  asm("mad.wide.u32 %0, %1, 1, %2;" : "=l"(r) : "r"(q), "l"(acc));
  return r;
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

// Block-wide sums of NU uint64 and ND double values with one barrier: each warp's lane 0
// writes its partials into the slot set `par`, which alternates between calls, so a call
// never overwrites slots that a thread may still be reading from the call before (every
// thread has left that call's reads before it reaches this call's barrier).
// Slots per set: at most PLAN_RED_U uint64 and PLAN_RED_D double values per reduction (kept
// small: with a staged Wan-sized row, three rows per SM fit in shared memory only so).
constexpr int PLAN_RED_U = 3, PLAN_RED_D = 1;
// Three staged rows per SM: each block holds the staged prefix, its static shared memory
// (the reduction slots, the staging barrier and the Philox word, 16-byte aligned) and the
// 1 KB the system reserves per block, within the SM's 228 KB.
static_assert(3 * (PLAN_STAGE_FLOAT4S * 16 +
                   ((2 * PLAN_RED_U * PLAN_WARPS * 8 + 2 * PLAN_RED_D * PLAN_WARPS * 8 + 8 + 4 + 15) / 16) * 16 +
                   1024) <= 228 * 1024,
              "the staged prefix no longer leaves room for three planner rows per SM");

template <int NU, int ND>
AB_DEV void block_sums(uint64_t (&u)[NU], double (&dv)[ND], uint64_t* ru, double* rd, int& par) {
  static_assert(NU <= PLAN_RED_U && ND <= PLAN_RED_D, "reduction slots");
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
#pragma unroll
    for (int k = 0; k < NU; ++k) u[k] += __shfl_xor_sync(0xffffffffu, u[k], o);
#pragma unroll
    for (int k = 0; k < ND; ++k) dv[k] += __shfl_xor_sync(0xffffffffu, dv[k], o);
  }
  uint64_t* su = ru + par * PLAN_RED_U * PLAN_WARPS;
  double* sd = rd + par * PLAN_RED_D * PLAN_WARPS;
  if (l == 0) {
#pragma unroll
    for (int k = 0; k < NU; ++k) su[k * PLAN_WARPS + w] = u[k];
#pragma unroll
    for (int k = 0; k < ND; ++k) sd[k * PLAN_WARPS + w] = dv[k];
  }
  __syncthreads();
  // the 16 warp partials: lane l (and l + 16) takes warp l's, then a 16-lane shuffle tree
  static_assert(PLAN_WARPS == 16, "one warp partial per half-warp lane");
#pragma unroll
  for (int k = 0; k < NU; ++k) u[k] = su[k * PLAN_WARPS + (l & 15)];
#pragma unroll
  for (int k = 0; k < ND; ++k) dv[k] = sd[k * PLAN_WARPS + (l & 15)];
#pragma unroll
  for (int o = 8; o; o >>= 1) {
#pragma unroll
    for (int k = 0; k < NU; ++k) u[k] += __shfl_xor_sync(0xffffffffu, u[k], o);
#pragma unroll
    for (int k = 0; k < ND; ++k) dv[k] += __shfl_xor_sync(0xffffffffu, dv[k], o);
  }
  par ^= 1;
}

// Exclusive scans in thread order of two uint64 values with one barrier (slot sets as above);
// returns this thread's prefixes and the block totals.
AB_DEV void block_exscan2_1b(uint64_t v0, uint64_t v1, uint64_t* ru, int& par, uint64_t& before0,
                             uint64_t& before1, uint64_t& total0, uint64_t& total1) {
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
  static_assert(PLAN_RED_U >= 2, "two scans per set");
  uint64_t* su = ru + par * PLAN_RED_U * PLAN_WARPS;
  if (l == 31) {
    su[w] = inc0;
    su[PLAN_WARPS + w] = inc1;
  }
  __syncthreads();
  // the 16 warp totals: lane l (and l + 16) takes warp l's, an inclusive 16-lane scan, then
  // the scan at lane w - 1 is what the warps before this one hold, at lane 15 the total
  uint64_t x0 = su[l & 15], x1 = su[PLAN_WARPS + (l & 15)];
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) {
    const uint64_t y0 = __shfl_up_sync(0xffffffffu, x0, o, 16);
    const uint64_t y1 = __shfl_up_sync(0xffffffffu, x1, o, 16);
    if ((l & 15) >= o) {
      x0 += y0;
      x1 += y1;
    }
  }
  const uint64_t p0 = __shfl_sync(0xffffffffu, x0, w > 0 ? w - 1 : 0);
  const uint64_t p1 = __shfl_sync(0xffffffffu, x1, w > 0 ? w - 1 : 0);
  total0 = __shfl_sync(0xffffffffu, x0, 15);
  total1 = __shfl_sync(0xffffffffu, x1, 15);
  before0 = (w > 0 ? p0 : 0ull) + inc0 - v0;
  before1 = (w > 0 ? p1 : 0ull) + inc1 - v1;
  par ^= 1;
}

// MODE 1: the whole row is staged in shared memory; MODE 2: its first PLAN_STAGE_FLOAT4S
// float4s are, and the rest is read from global memory on every pass.
template <int MODE>
__global__ void __launch_bounds__(PLAN_THREADS, 3) plan_kernel(PlanArgs a) {
  extern __shared__ float srow_smem[];
  __shared__ uint64_t ru[2 * PLAN_RED_U * PLAN_WARPS];
  __shared__ double rd[2 * PLAN_RED_D * PLAN_WARPS];
  __shared__ uint64_t row_bar;  // bulk staging of the row
  __shared__ uint32_t row_U;    // the row's Philox draw
  int par = 0;  // reduction slot set
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0)  // one thread draws; the others read it after the reductions' barriers
    row_U = philox4x32_10_w0(plan_counter_row(a, row), (uint32_t)a.offset, (uint32_t)(a.offset >> 32), 0u,
                             (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
  const int nK = a.nK;
  const float* grow = a.S + (size_t)row * nK;
  const bool uniform = a.mode == AB_PLAN_UNIFORM;
  const int nK4 = (nK + 3) >> 2;  // the row in whole float4s (zeros past nK)
  const uint64_t s = (uint64_t)a.s;
  const uint64_t target = s * TWO32;
  // This thread's contiguous chunk of float4s, in thread order; every pass after staging
  // walks it.  The first nK4 % PLAN_THREADS threads take one float4 more, so every thread
  // has work (an odd count keeps eight consecutive threads' 16-byte shared loads on
  // distinct banks; the even ones conflict two ways, which costs less than idle lanes).
  const int base4 = nK4 / PLAN_THREADS, rem4 = nK4 - base4 * PLAN_THREADS;
  const int c0 = tid * base4 + min(tid, rem4), c1 = c0 + base4 + (tid < rem4 ? 1 : 0);
  // The row's first ns4 float4s are staged in shared memory (all of it in MODE 1); the rest
  // is read from global memory, 16 bytes at a time when the row is 16-byte aligned and a
  // whole number of float4s.
  const int ns4 = MODE == 1 ? nK4 : min(nK4, PLAN_STAGE_FLOAT4S);
  const bool gvec = !uniform && ((uintptr_t)grow & 15u) == 0 && (nK & 3) == 0;
  auto gload4 = [&](int i) -> float4 {
    if (gvec) return __ldg(reinterpret_cast<const float4*>(grow) + i);
    float4 v;
    const int j = 4 * i;
    if (uniform) {
      v = make_float4(j < nK ? 1.f : 0.f, j + 1 < nK ? 1.f : 0.f, j + 2 < nK ? 1.f : 0.f,
                      j + 3 < nK ? 1.f : 0.f);
    } else {
      v.x = (j < nK) ? __ldg(grow + j) : 0.f;
      v.y = (j + 1 < nK) ? __ldg(grow + j + 1) : 0.f;
      v.z = (j + 2 < nK) ? __ldg(grow + j + 2) : 0.f;
      v.w = (j + 3 < nK) ? __ldg(grow + j + 3) : 0.f;
    }
    return v;
  };
  // Every pass walks this thread's chunk: its staged part from shared memory, then the rest.
  const int cm = min(max(ns4, c0), c1);
  auto walk = [&](auto&& body) {
    if (MODE == 1) {
      for (int i = c0; i < c1; ++i) body(i, reinterpret_cast<const float4*>(srow_smem)[i]);
    } else {
      for (int i = c0; i < cm; ++i) body(i, reinterpret_cast<const float4*>(srow_smem)[i]);
      for (int i = cm; i < c1; ++i) body(i, gload4(i));
    }
  };

  // This thread's part of F(lam): its saturated count and the sum of its other q_j.
  auto eval_part = [&](float lam, uint32_t& ns, uint64_t& qs) {
    if (lam < LAM_FAST_MAX) {
      const float L = __fmul_rn(lam, TWO32F);
      uint64_t acc = 0;
      float nsf = 0.f;
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float y = __fmul_rn(L, x4[k]);
          acc = add_wide(acc, f2u_rz(y));
          nsf += sat_flag(y);
        }
      });
      ns = (uint32_t)nsf;
      qs = acc - (uint64_t)ns * 0xFFFFFFFFull;
    } else {
      uint32_t n = 0;
      uint64_t q64 = 0;
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t q;
          n += fixed_q32(lam, x4[k], q);
          q64 += q;
        }
      });
      ns = n;
      qs = q64;
    }
  };

  // ---- positive blocks and their total score (fewer than s positive blocks = budget
  // unreachable); per-thread sums in compensated fp32, block sum in fp64.  With the row
  // staged in shared memory this pass also copies it there (coalesced, strided).
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
    const bool bulk = !uniform && ((uintptr_t)grow & 15u) == 0 && (nK & 3) == 0;
    if (bulk) {
      // the whole row in one bulk copy (one request in flight instead of a dependent
      // chain of loads per thread), then the sums over this thread's chunk
      if (tid == 0) {
        mbar_init(&row_bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&row_bar, (uint32_t)ns4 * 16u);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(srow_smem)),
            "l"(grow), "r"((uint32_t)ns4 * 16u), "r"(smem_u32(&row_bar))
            : "memory");
      }
      __syncthreads();  // the barrier is initialised before anyone waits on it
      const bool landed = mbar_wait_quiet(&row_bar, 0, kPlanTimeoutNs);
      if (__syncthreads_or(!landed)) {
        if (tid == 0) ab_flag(AB_ERR_DEVICE_TIMEOUT);
        return;
      }
      walk([&](const int i, const float4 v) {
        acc(v.x);
        acc(v.y);
        acc(v.z);
        acc(v.w);
      });
    } else {
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
        if (j < ns4) s4[j] = v;
        acc(v.x);
        acc(v.y);
        acc(v.z);
        acc(v.w);
      }
      // read by other threads only after the barrier of the block sum below
    }
    tot = (double)sum - (double)comp;
  }
  {
    uint64_t u1[1] = {npos};
    double d1[1] = {tot};
    block_sums<1, 1>(u1, d1, ru, rd, par);
    npos = u1[0];
    tot = d1[0];
  }
  const bool reachable = npos >= s;

  // ---- lambda*: the smallest positive fp32 (bit pattern in (0, 0x7F800000]) with
  // F(lambda) >= s 2^32.  F is monotone in the bit pattern, so any search that brackets the
  // boundary between lo (F < target, or lo = 0) and hi (F >= target, or hi = +inf, where
  // F = |positive| 2^32 >= target) and bisects finds the same lambda as a full 31-step
  // bisection.  An evaluation also leaves this thread's part of F -- its saturated count and
  // the sum of its other q_j -- which the output needs at lambda*.
  //
  // First pass: F at the three fp32 neighbours b0 - 1, b0, b0 + 1 of lambda0 = s / sum(S)
  // (and the sum of the scores unsaturated at b0).  Without saturation F(lambda) is
  // 2^32 lambda sum(S) less the truncations (under nK units, far below the 2^32 lambda ulp
  // sum(S) that one fp32 step adds), so lambda* is b0 or b0 + 1 and this one pass brackets it.
  uint32_t lo = 0u, hi = 0x7F800000u;
  bool hi_known = false;  // whether (hi_nsat, hi_q) hold this thread's part of F(hi)
  uint32_t hi_nsat = 0;
  uint64_t hi_q = 0;
  if (reachable) {
    const float lam0 = (tot > 0.0) ? (float)((double)a.s / tot) : 0.f;
    uint32_t b0 = __float_as_uint(lam0);
    if (!(lam0 > 0.f) || !isfinite(lam0)) b0 = 0x3F800000u;  // 1.0: any start works
    b0 = min(max(b0, 2u), 0x7F7FFFFEu);                       // three finite positive neighbours
    const float l3[3] = {__uint_as_float(b0 - 1u), __uint_as_float(b0), __uint_as_float(b0 + 1u)};
    uint32_t ns[3] = {0u, 0u, 0u};
    uint64_t qs[3] = {0ull, 0ull, 0ull};
    float rest = 0.f;
    if (l3[2] < LAM_FAST_MAX) {  // block-uniform; see sat_flag above
      float L3[3], nsf[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 3; ++c) L3[c] = __fmul_rn(l3[c], TWO32F);
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            const float y = __fmul_rn(L3[c], x4[k]);
            const float sat = sat_flag(y);
            qs[c] = add_wide(qs[c], f2u_rz(y));
            nsf[c] += sat;
            // scores unsaturated at b0: x (positive) times 1 - sat; NaN and x <= 0 add 0
            if (c == 1) rest = fmaf(1.f - sat, fmaxf(x4[k], 0.f), rest);
          }
        }
      });
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        ns[c] = (uint32_t)nsf[c];
        qs[c] -= (uint64_t)ns[c] * 0xFFFFFFFFull;  // the saturated blocks' 2^32 - 1 each
      }
    } else {
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            uint32_t q;
            const bool sat = fixed_q32(l3[c], x4[k], q);  // q = 0 when saturated
            ns[c] += sat;
            qs[c] += q;
            if (c == 1 && !sat && x4[k] > 0.f) rest += x4[k];
          }
        }
      });
    }
    uint64_t f3[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) f3[c] = ((uint64_t)ns[c] << 32) + qs[c];  // per thread below 2^39
    double r1[1] = {(double)rest};
    block_sums<3, 1>(f3, r1, ru, rd, par);
    // F is monotone: lo / hi from the three points
    int kstar = 3;  // first candidate with F >= target
#pragma unroll
    for (int c = 2; c >= 0; --c)
      if (f3[c] >= target) kstar = c;
    if (kstar < 3) {
      hi = b0 - 1u + (uint32_t)kstar;
      hi_nsat = kstar == 0 ? ns[0] : (kstar == 1 ? ns[1] : ns[2]);  // kstar is block-uniform
      hi_q = kstar == 0 ? qs[0] : (kstar == 1 ? qs[1] : qs[2]);
      hi_known = true;
    }
    bool lo_set = kstar > 0;  // F(lo) < target was evaluated (else lo = 0, F(0) = 0)
    if (lo_set) lo = b0 - 2u + (uint32_t)kstar;
    if (hi - lo > 1u && r1[0] > 0.0) {
      // Newton on the exact integer sum from b0: F grows by about (sum of the unsaturated
      // scores) 2^32 per unit lambda (the water-filling update).
      const double lam_n = (double)l3[1] + ((double)target - (double)f3[1]) / (r1[0] * 4294967296.0);
      const float lf = (float)lam_n;
      const uint32_t b2 = __float_as_uint(lf);
      if (lf > 0.f && isfinite(lf) && b2 > lo && b2 < hi) {
        uint64_t f1[1];
        uint32_t ns2;
        uint64_t qs2;
        eval_part(lf, ns2, qs2);
        f1[0] = ((uint64_t)ns2 << 32) + qs2;
        double none[1] = {0.0};
        block_sums<1, 1>(f1, none, ru, rd, par);
        if (f1[0] >= target) {
          hi = b2;
          hi_nsat = ns2;
          hi_q = qs2;
          hi_known = true;
        } else {
          lo = b2;
          lo_set = true;
        }
      }
    }
    // the rest (rare): doubling steps away from the evaluated side until the other side is
    // evaluated too (lambda = +inf and lambda = 0 are the outer bounds), then bisection
    uint32_t step = 1;
    while (hi - lo > 1u) {
      uint32_t cand;
      if (!hi_known) {  // step up from lo
        cand = (0x7F800000u - lo > step) ? lo + step : 0x7F800000u;
        step <<= 1;
      } else if (!lo_set) {  // step down from hi
        if (hi <= step) {    // reached lambda = 0: bisect [0, hi]
          lo = 0u;
          lo_set = true;
          continue;
        }
        cand = hi - step;
        step <<= 1;
      } else {
        cand = lo + ((hi - lo) >> 1);
      }
      uint32_t ns2;
      uint64_t qs2;
      eval_part(__uint_as_float(cand), ns2, qs2);
      uint64_t f1[1] = {((uint64_t)ns2 << 32) + qs2};
      double none[1] = {0.0};
      block_sums<1, 1>(f1, none, ru, rd, par);
      if (f1[0] >= target) {
        hi = cand;
        hi_nsat = ns2;
        hi_q = qs2;
        hi_known = true;
      } else {
        lo = cand;
        lo_set = true;
      }
    }
    if (!hi_known) eval_part(__uint_as_float(hi), hi_nsat, hi_q);  // lambda* = +inf (pathological rows)
  }
  const float lam = __uint_as_float(hi);

  // ---- this thread's chunk: saturated count and the sum of its other q_j (budget
  // reachable: the part of F(lambda*) kept above), or (budget unreachable) its positive
  // blocks (pi = 1) and its other blocks (the first s - |positive| of them complete the draw)
  uint64_t my_sat, my_rest;
  if (reachable) {
    my_sat = hi_nsat;
    my_rest = hi_q;
  } else {
    my_sat = 0;
    my_rest = 0;
    walk([&](const int i, const float4 v) {
      const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (4 * i + k >= nK) break;
        if (x4[k] > 0.f) ++my_sat; else ++my_rest;
      }
    });
  }
  uint64_t sat_before, rest_before, n_sat, tot_rest;
  block_exscan2_1b(my_sat, my_rest, ru, par, sat_before, rest_before, n_sat, tot_rest);

  const uint32_t U = row_U;  // written before the first barrier
  // lattice points U + k 2^32 below x, for 0 <= x <= s 2^32 (U < 2^32)
  const uint64_t CB = TWO32 - 1u - (uint64_t)U;
  auto below = [&](uint64_t x) -> uint64_t { return (x + CB) >> 32; };
  // Saturated blocks come first in the layout, block k of them covering [k 2^32, (k+1) 2^32):
  // each holds exactly one lattice point, so every saturated block is drawn.  The other
  // blocks follow in ascending order; this thread's chunk covers [start, start + my_rest).
  // The intervals of the threads before this one are contiguous, so the draws before this
  // thread's first output are its predecessors' saturated blocks plus the lattice points in
  // [n_sat 2^32, start).  With the budget unreachable, the first s - n_sat zero blocks (in
  // order) complete the draw.
  const uint64_t start = n_sat * TWO32 + rest_before;
  const uint64_t need = s - min(n_sat, s);
  const uint64_t base = n_sat * TWO32;
  const uint64_t out_before =
      sat_before + (reachable ? below(min(start, target)) - below(min(base, target)) : min(rest_before, need));
  const uint64_t n_sel =
      n_sat + (reachable ? below(min(base + tot_rest, target)) - below(min(base, target)) : min(tot_rest, need));
  if (n_sel != s && tid == 0) ab_flag(AB_ERR_DEVICE_CHECK);  // cannot happen; guards the writes

  // ---- write ascending idx and the fixed-point probability (its log follows below)
  {
    // Below the cap s 2^32, a non-saturated block [pos, pos + q) holds a lattice point iff
    // dist < q, with dist = (U - pos) mod 2^32 the distance to the next point, and the next
    // block starts at distance (dist - q) mod 2^32: 32-bit arithmetic.  The chunk that
    // reaches the cap clips its intervals at s 2^32 (64-bit positions).
    const bool capped = reachable && start + my_rest > target;
    uint32_t dist = U - (uint32_t)start;
    uint64_t pos = start, zero_i = rest_before;
    uint64_t o = out_before;
    int32_t* oidx = a.idx + (size_t)row * a.s;
    uint32_t* oraw = reinterpret_cast<uint32_t*>(a.logpi + (size_t)row * a.s);
    if (reachable && !capped && lam < LAM_FAST_MAX) {
      // the common case, branch-light, with the FMA-pipe form of q (see sat_flag): a
      // saturated block has q = 0 here and is drawn; a block past the row's end (score 0,
      // q = 0) never is
      uint32_t o32 = (uint32_t)out_before;
      const uint32_t s32 = (uint32_t)a.s;
      const float L = __fmul_rn(lam, TWO32F);
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float y = __fmul_rn(L, x4[k]);
          const bool sat = y >= TWO32F;
          const uint32_t q = f2u_rz(sat ? 0.f : y);
          const bool sel = sat || dist < q;
          dist -= q;
          if (sel) {
            if (o32 < s32) {
              oidx[o32] = 4 * i + k;
              oraw[o32] = sat ? 0xFFFFFFFFu : q;  // pi = 1, or q (at most 2^32 - 256)
            }
            ++o32;
          }
        }
      });
    } else if (reachable && !capped) {
      // the same with the integer form of q (lambda >= 2^95)
      uint32_t o32 = (uint32_t)out_before;
      const uint32_t s32 = (uint32_t)a.s;
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t q;
          const bool sat = fixed_q32(lam, x4[k], q);
          const bool sel = sat || dist < q;
          dist -= q;
          if (sel) {
            if (o32 < s32) {
              oidx[o32] = 4 * i + k;
              oraw[o32] = sat ? 0xFFFFFFFFu : q;  // pi = 1, or q (at most 2^32 - 256)
            }
            ++o32;
          }
        }
      });
    } else {
      walk([&](const int i, const float4 v) {
        const float x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int j = 4 * i + k;
          if (j >= nK) break;
          bool sel;
          uint32_t qq = 0xFFFFFFFFu;  // pi = 1 (a capped or ordinary q is at most 2^32 - 256)
          if (reachable) {
            uint32_t q;
            if (fixed_q32(lam, x4[k], q)) {
              sel = true;
            } else if (!capped) {
              sel = dist < q;
              qq = q;
              dist -= q;
            } else {
              const uint64_t st = min(pos, target), en = min(pos + q, target);
              sel = below(en) != below(st);
              qq = (uint32_t)(en - st);
              pos += q;
            }
          } else {
            sel = (x4[k] > 0.f) || (zero_i++ < need);
          }
          if (sel) {
            if (o < s) {
              oidx[o] = j;
              oraw[o] = qq;
            }
            ++o;
          }
        }
      });
    }
  }
  // log(pi) for the s outputs, spread evenly over the threads (no divergent fp64 log)
  __syncthreads();
  {
    float* olp = a.logpi + (size_t)row * a.s;
    uint32_t* raw = reinterpret_cast<uint32_t*>(olp);
    constexpr int LB = 4;  // outputs per batch: their loads are in flight together
    for (int o0 = tid; o0 < a.s; o0 += LB * PLAN_THREADS) {
      uint32_t q[LB];
#pragma unroll
      for (int k = 0; k < LB; ++k) {
        const int o = o0 + k * PLAN_THREADS;
        q[k] = o < a.s ? raw[o] : 0xFFFFFFFFu;
      }
#pragma unroll
      for (int k = 0; k < LB; ++k) {
        const int o = o0 + k * PLAN_THREADS;
        if (o < a.s)
          olp[o] = (q[k] == 0xFFFFFFFFu || a.mode == AB_PLAN_SIP_NO_IPW)
                       ? 0.f
                       : (float)log((double)q[k] * (1.0 / 4294967296.0));
      }
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
