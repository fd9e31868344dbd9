// IBCS selector for sm_100a: pooled keys, intra-block k-means, block scores.
//
// AB-Attention page (onedev.kr/papers/1521), section "how it differs": queries are
// cut into 128-token blocks and keys/values into small blocks (4 tokens on the page);
// inside each query block one k-means iteration forms 8 query clusters with centroids
// and query shares; each KV block is scored by the share-weighted softmax mass of the
// centroids over the pooled keys.  Ablation paragraph: 16-query positional segment
// means, used here as the k-means start (and alone with zero iterations).
//
// Exactness: pooled keys and centroids are rounded once to bf16 from fp64 means (sums
// of at most 128 bf16 values are exact in fp64, the division is IEEE), so they equal
// the CPU reference bit for bit; assignments use fp64 distances.  Logits use the bf16
// operands with fp32 accumulation; softmax statistics are fp32 in the log2 domain.
//
//   pool_kernel      Kp[bh, j, :]  = bf16(mean of block j's valid keys)
//   kmeans_kernel    per (bh, query block): centroids (bf16) and shares (fp32)
//   score_tc_kernel<1>  per centroid row: running max m and sum Z of exp2(logit - m)
//   score_tc_kernel<2>  S[bh, i, j] = sum_c (w_c / Z_c) exp2(logit_cj - m_c)
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int CMAX = 8;          // centroid slots per query block
constexpr int KM_THREADS = 256;

struct SelectArgs {
  const uint16_t* Q;
  const uint16_t* K;
  uint16_t* Kp;      // [BH, nK, D]
  uint16_t* cent;    // [BH, nQ, CMAX, D]
  float* w;          // [BH, nQ, CMAX]
  float* stats;      // [BH, nQ, CMAX, 2]  (m in log2 units, Z)
  float* S;          // [BH, nQ, nK]
  int8_t* labels;    // optional [BH, nQ*128]
  int BH, N, nQ, nK, bk, C, iters;
  float scale_log2;  // log2(e) / sqrt(d)
};

AB_DEV double bf16_to_double(uint16_t b) { return (double)bf16_bits_to_float(b); }

// ------------------------------------------------------------------ pooled keys

template <int D>
__global__ void pool_kernel(SelectArgs a) {
  constexpr int UNITS = D / 8;
  const size_t total = (size_t)a.BH * a.nK * UNITS;
  for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const int u = (int)(g % UNITS);
    const size_t bj = g / UNITS;  // bh * nK + j
    const int j = (int)(bj % a.nK);
    const size_t bh = bj / a.nK;
    const int t0 = j * a.bk, t1 = min(a.N, t0 + a.bk);
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const uint16_t* src = a.K + (bh * a.N + t0) * D + u * 8;
    for (int t = t0; t < t1; ++t, src += D) {
      const uint4 v = __ldg((const uint4*)src);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_to_double((uint16_t)(w4[e] & 0xffffu));
        acc[2 * e + 1] += bf16_to_double((uint16_t)(w4[e] >> 16));
      }
    }
    const double cnt = (double)(t1 - t0);
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = (uint32_t)bf16_bits_from_double(acc[2 * e] / cnt) |
             ((uint32_t)bf16_bits_from_double(acc[2 * e + 1] / cnt) << 16);
    *(uint4*)(a.Kp + bj * D + u * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ k-means
//
// One CTA of 256 threads per (bh, query block).
//  * Segment means (the start) and member means (the update) are exact fp64 sums of the
//    bf16 rows divided by the count (IEEE division), as the CPU reference computes them.
//    The update visits the rows in label order (a counting sort), so each thread (one
//    dimension) runs through the rows once, accumulating into the current cluster.
//  * Assignment: two threads per row compute the 8 squared distances in fp32 against the
//    fp32-rounded centroids.  With u = 2^-24 and n = d terms, the fp32 distance differs
//    from the exact one by at most (n + 4) u (2 |q|^2 + 2 |c|^2) (rounding of c, of q - c,
//    and of the n-term sum), so when the best and second-best fp32 distances are further
//    apart than the sum of their bounds the fp32 choice is the exact argmin.  Rows inside
//    the margin are recomputed in fp64 (ties to the lowest cluster), like the reference.

template <int D>
__global__ void __launch_bounds__(KM_THREADS) kmeans_kernel(SelectArgs a) {
  __shared__ __align__(16) uint16_t qs[128 * D];
  __shared__ double c64[CMAX * D];
  __shared__ __align__(16) float cf[CMAX * D];
  __shared__ float c2[CMAX];
  __shared__ int cnt[CMAX];
  __shared__ int off[CMAX];
  __shared__ int alive[CMAX];
  __shared__ int8_t lab[128];
  __shared__ uint8_t perm[128];
  const int bq = blockIdx.x;  // bh * nQ + i
  const int bh = bq / a.nQ, i = bq - bh * a.nQ;
  const int row0 = i * 128;
  const int n = min(128, a.N - row0);
  const int tid = threadIdx.x;
  const int C = a.C;
  constexpr int UNITS = D / 8;
  constexpr int H = D / 2;  // dimensions per thread in the assignment

  const uint16_t* qsrc = a.Q + ((size_t)bh * a.N + row0) * D;
  for (int e = tid; e < n * UNITS; e += KM_THREADS) ((uint4*)qs)[e] = __ldg((const uint4*)qsrc + e);
  if (tid < CMAX) {
    const int s0 = tid * n / C, s1 = (tid + 1) * n / C;
    cnt[tid] = (tid < C) ? s1 - s0 : 0;
    alive[tid] = (tid < C) && (s1 > s0);
  }
  if (tid < 128) {
    int c = -1;
    if (tid < n)
      for (int cc = 0; cc < C; ++cc)
        if (tid >= cc * n / C && tid < (cc + 1) * n / C) c = cc;
    lab[tid] = (int8_t)c;
  }
  __syncthreads();
  // segment means (fp64, exact sums)
  for (int p = tid; p < CMAX * D; p += KM_THREADS) {
    const int c = p / D, dd = p - c * D;
    double acc = 0.0;
    if (c < C) {
      const int s0 = c * n / C, s1 = (c + 1) * n / C;
      for (int r = s0; r < s1; ++r) acc += bf16_to_double(qs[r * D + dd]);
      if (s1 > s0) acc = acc / (double)(s1 - s0);
    }
    c64[p] = acc;
  }
  __syncthreads();

  const int ar = tid >> 1;   // assignment: row
  const int ah = tid & 1;    // ... and which half of the dimensions
  for (int it = 0; it < a.iters; ++it) {
    // fp32 copies of the centroids and their squared norms
    for (int p = tid; p < CMAX * D; p += KM_THREADS) cf[p] = (float)c64[p];
    __syncthreads();
    if (tid < 32) {
#pragma unroll
      for (int c = 0; c < CMAX; ++c) {
        float part = 0.f;
        for (int dd = tid; dd < D; dd += 32) part = fmaf(cf[c * D + dd], cf[c * D + dd], part);
#pragma unroll
        for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (tid == 0) c2[c] = part;
      }
    }
    __syncthreads();
    // assignment (rows >= n take part in the shuffles but are not stored)
    {
      const uint16_t* qrow = qs + (ar < n ? ar : 0) * D + ah * H;
      float dist[CMAX];
#pragma unroll
      for (int c = 0; c < CMAX; ++c) dist[c] = 0.f;
      float q2 = 0.f;
#pragma unroll 4
      for (int e = 0; e < H; e += 8) {
        const uint4 v = *(const uint4*)(qrow + e);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        float qv[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          qv[2 * k] = __uint_as_float(w4[k] << 16);
          qv[2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) q2 = fmaf(qv[k], qv[k], q2);
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
          const float* cc = cf + c * D + ah * H + e;
          const float4 c0 = *(const float4*)cc;
          const float4 c1 = *(const float4*)(cc + 4);
          const float dv[8] = {qv[0] - c0.x, qv[1] - c0.y, qv[2] - c0.z, qv[3] - c0.w,
                               qv[4] - c1.x, qv[5] - c1.y, qv[6] - c1.z, qv[7] - c1.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) dist[c] = fmaf(dv[k], dv[k], dist[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < CMAX; ++c) dist[c] += __shfl_xor_sync(0xffffffffu, dist[c], 1);
      q2 += __shfl_xor_sync(0xffffffffu, q2, 1);
      int best = -1, second = -1;
      float d1 = 0.f, d2 = 0.f, n1 = 0.f, n2 = 0.f;  // best / second distance and |c|^2
#pragma unroll
      for (int c = 0; c < CMAX; ++c) {
        if (!alive[c]) continue;
        if (best < 0 || dist[c] < d1) {
          second = best; d2 = d1; n2 = n1;
          best = c; d1 = dist[c]; n1 = c2[c];
        } else if (second < 0 || dist[c] < d2) {
          second = c; d2 = dist[c]; n2 = c2[c];
        }
      }
      constexpr float U = 5.9604645e-8f;  // 2^-24
      bool certain = true;
      if (second >= 0) {
        const float kb = (float)(D + 4) * U * 2.f * 1.0625f;  // bound factor with margin
        certain = d2 - d1 > kb * ((q2 + n1) + (q2 + n2));
      }
      // rows whose fp32 margin is too small: recompute all distances in fp64
      if (__any_sync(0xffffffffu, !certain && ar < n)) {
        double dd64[CMAX];
#pragma unroll
        for (int c = 0; c < CMAX; ++c) dd64[c] = 0.0;
        if (!certain) {
          for (int e = 0; e < H; ++e) {
            const double qd = bf16_to_double(qrow[e]);
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
              const double dv = qd - c64[c * D + ah * H + e];
              dd64[c] = fma(dv, dv, dd64[c]);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < CMAX; ++c) dd64[c] += __shfl_xor_sync(0xffffffffu, dd64[c], 1);
        if (!certain) {
          best = -1;
          double b64 = 0.0;
#pragma unroll
          for (int c = 0; c < CMAX; ++c)
            if (alive[c] && (best < 0 || dd64[c] < b64)) { best = c; b64 = dd64[c]; }
        }
      }
      if (ah == 0 && ar < n) lab[ar] = (int8_t)best;
    }
    if (tid < CMAX) cnt[tid] = 0;
    __syncthreads();
    if (tid < n) atomicAdd(&cnt[lab[tid]], 1);
    __syncthreads();
    if (tid == 0) {
      int o = 0;
      for (int c = 0; c < CMAX; ++c) { off[c] = o; o += cnt[c]; }
    }
    __syncthreads();
    if (tid < n) perm[atomicAdd(&off[lab[tid]], 1)] = (uint8_t)tid;  // off[c] ends at its cluster's end
    __syncthreads();
    // update: each thread owns a dimension and walks the rows grouped by cluster
    if (tid < D) {
      int r0 = 0;
      for (int c = 0; c < CMAX; ++c) {
        const int k = cnt[c];
        if (k > 0) {
          double acc = 0.0;
          for (int q = r0; q < r0 + k; ++q) acc += bf16_to_double(qs[perm[q] * D + tid]);
          c64[c * D + tid] = acc / (double)k;
        }
        r0 += k;
      }
    }
    __syncthreads();
    if (tid < CMAX) alive[tid] = cnt[tid] > 0;
    __syncthreads();
  }

  // outputs: bf16 centroids (zero when empty) and shares
  uint16_t* cdst = a.cent + (size_t)bq * CMAX * D;
  for (int p = tid; p < CMAX * D; p += KM_THREADS) {
    const int c = p / D;
    cdst[p] = alive[c] ? bf16_bits_from_double(c64[p]) : (uint16_t)0;
  }
  if (tid < CMAX) a.w[(size_t)bq * CMAX + tid] = alive[tid] ? (float)((double)cnt[tid] / (double)n) : 0.f;
  if (a.labels && tid < 128) a.labels[(size_t)bh * a.nQ * 128 + row0 + tid] = (tid < n) ? lab[tid] : (int8_t)-1;
}

// ------------------------------------------------------------------ block scores (tcgen05)
//
// The page's batched scoring ("premises & limits": query/KV blocks scored as batched
// matrix operations) as two tensor-core streaming passes per CTA of 16 query blocks
// (128 centroid rows), over all pooled keys of the head in tiles of 128:
//   PASS 1: D[centroid row, key] = C Kp^T  (A = centroids, B = key tile, both K-major).
//           Thread r (= TMEM lane r) keeps the running max m and sum Z of exp2(logit - m).
//   PASS 2: D[key, centroid col] = Kp C^T (A = key tile, B = centroids), so thread j owns
//           one KV block and sums (w_c / Z_c) exp2(logit - m_c) over the 8 columns of each
//           query block in registers; S rows are stored coalesced.
// Roles as in the attention kernel: warps 0-3 consume TMEM, warps 4-7 stream tiles with
// cp.async (2 stages), warp 8 allocates TMEM and issues the MMAs.

constexpr int SCT_THREADS = 288;

template <int D>
struct ScoreSmem {
  static constexpr uint32_t TILE = 128u * D * 2u;
  static constexpr uint32_t CHUNK = 128u * 128u;
  static constexpr int STAGES = 2;
  static constexpr uint32_t FIX_OFF = 0;  // centroid tile
  static constexpr uint32_t KP_OFF = FIX_OFF + TILE;
  static constexpr uint32_t COL_OFF = KP_OFF + STAGES * TILE;  // pass 2: m[128], coef[128]
  static constexpr uint32_t BAR_OFF = COL_OFF + 2u * 128u * 4u;
  // CFULL, FULL[2], EMPTY[2], SFULL[2], SFREE[2], DRAIN
  static constexpr uint32_t NBARS = 10;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBARS * 8u;
  static constexpr uint32_t BYTES = MISC_OFF + 16u;
  static constexpr uint32_t ALLOC = BYTES + 1024u;
};

enum { SB_CFULL = 0, SB_FULL0 = 1, SB_EMPTY0 = 3, SB_SFULL0 = 5, SB_SFREE0 = 7, SB_DRAIN = 9 };

// Two CTAs per SM (98 KB of shared memory and 256 TMEM columns each), so two consumer
// warpgroups interleave their exp2 work on the MUFU units.
template <int D, int PASS>
__global__ void __launch_bounds__(SCT_THREADS, 2) score_tc_kernel(SelectArgs a, uint64_t timeout_ns) {
  using L = ScoreSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF);
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF + 4);
  float2* col_mc = (float2*)(smem + L::COL_OFF);  // pass 2: (m, w/Z) per centroid column

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int groups = (a.nQ + 15) / 16;
  const int bh = blockIdx.x / groups;
  const int g = blockIdx.x - bh * groups;
  const int T = (a.nK + 127) / 128;

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars[SB_CFULL], 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[SB_FULL0 + b], 128);
      mbar_init(&bars[SB_EMPTY0 + b], 1);
      mbar_init(&bars[SB_SFULL0 + b], 1);
      mbar_init(&bars[SB_SFREE0 + b], 128);
    }
    mbar_init(&bars[SB_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------------- producers
    const int p = tid - 128, u = p & 15, rsub = p >> 4;
    constexpr int UNITS = D / 8;
    for (int r = rsub; r < 128; r += 8) {  // centroid rows: 16 query blocks x 8 slots
      if (u < UNITS) {
        const int qb = g * 16 + (r >> 3);
        const bool ok = qb < a.nQ;
        const uint16_t* src = a.cent + (((size_t)bh * a.nQ + (ok ? qb : 0)) * CMAX + (r & 7)) * D + u * 8;
        cp_async_16(sbase + L::FIX_OFF + (u >> 3) * L::CHUNK + sw128_off(r, u & 7), src, ok ? 16u : 0u);
      }
    }
    mbar_arrive_cpasync(&bars[SB_CFULL]);
    const uint16_t* kp = a.Kp + (size_t)bh * a.nK * D;
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (t >= 2 && !mbar_wait(&bars[SB_EMPTY0 + st], ((t >> 1) - 1) & 1, abort_flag, timeout_ns)) break;
      const uint32_t dst = sbase + L::KP_OFF + st * L::TILE;
      for (int r = rsub; r < 128; r += 8) {
        if (u < UNITS) {
          const int j = t * 128 + r;
          const bool ok = j < a.nK;
          cp_async_16(dst + (u >> 3) * L::CHUNK + sw128_off(r, u & 7),
                      kp + (size_t)(ok ? j : 0) * D + u * 8, ok ? 16u : 0u);
        }
      }
      mbar_arrive_cpasync(&bars[SB_FULL0 + st]);
    }
    cp_async_wait_all();
  } else if (warp == 8) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, 0, 0);
      bool ok = mbar_wait(&bars[SB_CFULL], 0, abort_flag, timeout_ns);
      for (int t = 0; t < T && ok; ++t) {
        const int st = t & 1;
        ok = mbar_wait(&bars[SB_FULL0 + st], (t >> 1) & 1, abort_flag, timeout_ns);
        if (ok && t >= 2) ok = mbar_wait(&bars[SB_SFREE0 + st], ((t >> 1) - 1) & 1, abort_flag, timeout_ns);
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t cbase = sbase + L::FIX_OFF;
        const uint32_t kbase = sbase + L::KP_OFF + st * L::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::CHUNK + (kk & 3) * 32;
          const uint64_t dc = sdesc_sw128(cbase + off, 16, 1024);
          const uint64_t dk = sdesc_sw128(kbase + off, 16, 1024);
          if (PASS == 1) umma_f16_ss(tmem + st * 128, dc, dk, IDESC, kk > 0 ? 1u : 0u);
          else umma_f16_ss(tmem + st * 128, dk, dc, IDESC, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[SB_SFULL0 + st]);
        umma_commit(&bars[SB_EMPTY0 + st]);
      }
      umma_commit(&bars[SB_DRAIN]);
      mbar_wait(&bars[SB_DRAIN], 0, abort_flag, timeout_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers (warps 0-3)
    const int r = tid;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (PASS == 2) {  // per-column constants: column r = (query block r>>3, slot r&7)
      const int qb = g * 16 + (r >> 3);
      float mm = 0.f, cf = 0.f;
      if (qb < a.nQ) {
        const size_t crow = ((size_t)bh * a.nQ + qb) * CMAX + (r & 7);
        const float Z = a.stats[crow * 2 + 1];
        mm = a.stats[crow * 2];
        cf = (Z > 0.f) ? a.w[crow] / Z : 0.f;
        if (!(mm > -INFINITY)) { mm = 0.f; cf = 0.f; }
      }
      col_mc[r] = make_float2(mm, cf);
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 consumer warps only
    }
    float m = -INFINITY, z = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      ok = mbar_wait(&bars[SB_SFULL0 + st], (t >> 1) & 1, abort_flag, timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sadr = tmem + st * 128 + lane_off;
      if (PASS == 1) {
        // online max / sum over 32-column chunks (keeps 32 values live)
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(sadr + c0, v);
          tmem_wait_ld();
          float mt = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float l = (t * 128 + c0 + c < a.nK) ? __uint_as_float(v[c]) * a.scale_log2 : -INFINITY;
            v[c] = __float_as_uint(l);
            mt = fmaxf(mt, l);
          }
          if (mt > m) {
            z = (m == -INFINITY) ? 0.f : z * fast_exp2(m - mt);
            m = mt;
          }
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < 32; ++c) acc += fast_exp2(__uint_as_float(v[c]) - m);
          z += acc;
        }
        tc_fence_before();
        mbar_arrive(&bars[SB_SFREE0 + st]);
      } else {
        const int j = t * 128 + r;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {  // 4 query blocks per TMEM load
          uint32_t v[32];
          tmem_ld_32x32b_x32(sadr + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              // re-read per tile (volatile): hoisting all 128 columns would need 256 registers
              float mm, cf;
              asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                           : "=f"(mm), "=f"(cf)
                           : "r"(smem_u32(col_mc + c0 + q * 8 + c)));
              acc = fmaf(cf, fast_exp2(fmaf(__uint_as_float(v[q * 8 + c]), a.scale_log2, -mm)), acc);
            }
            const int qb = g * 16 + (c0 >> 3) + q;
            if (j < a.nK && qb < a.nQ) a.S[((size_t)bh * a.nQ + qb) * a.nK + j] = acc;
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[SB_SFREE0 + st]);
      }
    }
    if (PASS == 1 && ok) {
      const int qb = g * 16 + (r >> 3);
      if (qb < a.nQ) {
        const size_t crow = ((size_t)bh * a.nQ + qb) * CMAX + (r & 7);
        a.stats[crow * 2] = m;
        a.stats[crow * 2 + 1] = z;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace abattn
