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
//   score_kernel<1>  per centroid row: running max m and sum Z of exp2(logit - m)
//   score_kernel<2>  S[bh, i, j] = sum_c (w_c / Z_c) exp2(logit_cj - m_c)
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int CMAX = 8;          // centroid slots per query block
constexpr int KM_THREADS = 256;
constexpr int SC_THREADS = 128;  // 16 query blocks x 8 centroid slots
constexpr int SC_KT = 32;        // pooled keys per shared-memory tile

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

template <int D>
__global__ void __launch_bounds__(KM_THREADS) kmeans_kernel(SelectArgs a) {
  __shared__ __align__(16) uint16_t qs[128 * D];
  __shared__ double c64[CMAX * D];
  __shared__ int cnt[CMAX];
  __shared__ int alive[CMAX];
  __shared__ int8_t lab[128];
  const int bq = blockIdx.x;  // bh * nQ + i
  const int bh = bq / a.nQ, i = bq - bh * a.nQ;
  const int row0 = i * 128;
  const int n = min(128, a.N - row0);
  const int tid = threadIdx.x;
  const int C = a.C;
  constexpr int UNITS = D / 8;

  const uint16_t* qsrc = a.Q + ((size_t)bh * a.N + row0) * D;
  for (int e = tid; e < n * UNITS; e += KM_THREADS)
    ((uint4*)qs)[e] = __ldg((const uint4*)qsrc + e);
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
  // segment means (fp64)
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

  for (int it = 0; it < a.iters; ++it) {
    // assignment: thread r owns query row r (kept in registers)
    if (tid < n) {
      uint32_t qr[D / 2];
#pragma unroll
      for (int e = 0; e < D / 8; ++e) {
        const uint4 v = ((const uint4*)(qs + tid * D))[e];
        qr[4 * e] = v.x; qr[4 * e + 1] = v.y; qr[4 * e + 2] = v.z; qr[4 * e + 3] = v.w;
      }
      double best = 0.0;
      int bc = -1;
      for (int c = 0; c < C; ++c) {
        if (!alive[c]) continue;
        const double* cc = c64 + c * D;
        double dist = 0.0;
#pragma unroll
        for (int e = 0; e < D / 2; ++e) {
          const double d0 = bf16_to_double((uint16_t)(qr[e] & 0xffffu)) - cc[2 * e];
          const double d1 = bf16_to_double((uint16_t)(qr[e] >> 16)) - cc[2 * e + 1];
          dist = fma(d0, d0, dist);
          dist = fma(d1, d1, dist);
        }
        if (bc < 0 || dist < best) { best = dist; bc = c; }
      }
      lab[tid] = (int8_t)bc;
    }
    __syncthreads();
    if (tid < CMAX) {
      int k = 0;
      for (int r = 0; r < n; ++r) k += (lab[r] == tid);
      cnt[tid] = k;
    }
    __syncthreads();
    // update: fp64 member means; empty clusters keep their previous centroid
    for (int p = tid; p < CMAX * D; p += KM_THREADS) {
      const int c = p / D, dd = p - c * D;
      if (cnt[c] > 0) {
        double acc = 0.0;
        for (int r = 0; r < n; ++r)
          if (lab[r] == c) acc += bf16_to_double(qs[r * D + dd]);
        c64[p] = acc / (double)cnt[c];
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

// ------------------------------------------------------------------ block scores (SIMT)

// PASS 1: per centroid row, running (max, sum of exp2) over all pooled keys.
// PASS 2: emit S.  CTA = 16 query blocks x 8 centroid slots = 128 rows, thread = row.
template <int D, int PASS>
__global__ void __launch_bounds__(SC_THREADS) score_kernel(SelectArgs a) {
  __shared__ __align__(16) float kt[SC_KT * D];
  __shared__ float sbuf[16][SC_KT + 1];
  const int groups = (a.nQ + 15) / 16;
  const int bh = blockIdx.x / groups;
  const int g = blockIdx.x - bh * groups;
  const int tid = threadIdx.x;
  const int ql = tid >> 3, c = tid & 7;
  const int qb = g * 16 + ql;
  const bool live = qb < a.nQ;
  const size_t crow = ((size_t)bh * a.nQ + (live ? qb : 0)) * CMAX + c;

  float cr[D];
  {
    const uint16_t* cs = a.cent + crow * D;
#pragma unroll
    for (int e = 0; e < D; e += 8) {
      const uint4 v = live ? __ldg((const uint4*)(cs + e)) : make_uint4(0, 0, 0, 0);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        cr[e + 2 * k] = bf16_bits_to_float((uint16_t)(w4[k] & 0xffffu));
        cr[e + 2 * k + 1] = bf16_bits_to_float((uint16_t)(w4[k] >> 16));
      }
    }
  }
  float m = -INFINITY, z = 0.f, coef = 0.f;
  if (PASS == 2 && live) {
    m = a.stats[crow * 2];
    const float Z = a.stats[crow * 2 + 1];
    const float wv = a.w[crow];
    coef = (Z > 0.f) ? wv / Z : 0.f;
  }
  const uint16_t* kp = a.Kp + (size_t)bh * a.nK * D;
  for (int j0 = 0; j0 < a.nK; j0 += SC_KT) {
    const int nk = min(SC_KT, a.nK - j0);
    __syncthreads();
    for (int e = tid; e < SC_KT * D / 2; e += SC_THREADS) {
      const int kk = e / (D / 2);
      uint32_t v = 0;
      if (kk < nk) v = __ldg((const uint32_t*)(kp + (size_t)(j0 + kk) * D) + (e - kk * (D / 2)));
      kt[2 * e] = bf16_bits_to_float((uint16_t)(v & 0xffffu));
      kt[2 * e + 1] = bf16_bits_to_float((uint16_t)(v >> 16));
    }
    __syncthreads();
    float l[SC_KT];
#pragma unroll
    for (int kk = 0; kk < SC_KT; ++kk) {
      const float4* kv = (const float4*)(kt + kk * D);
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D / 4; ++e) {
        const float4 x = kv[e];
        acc = fmaf(cr[4 * e], x.x, acc);
        acc = fmaf(cr[4 * e + 1], x.y, acc);
        acc = fmaf(cr[4 * e + 2], x.z, acc);
        acc = fmaf(cr[4 * e + 3], x.w, acc);
      }
      l[kk] = (kk < nk) ? acc * a.scale_log2 : -INFINITY;
    }
    if (PASS == 1) {
      float mt = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < SC_KT; ++kk) mt = fmaxf(mt, l[kk]);
      const float mn = fmaxf(m, mt);
      float acc = (m == -INFINITY) ? 0.f : z * fast_exp2(m - mn);
#pragma unroll
      for (int kk = 0; kk < SC_KT; ++kk) acc += fast_exp2(l[kk] - mn);
      z = acc;
      m = mn;
    } else {
#pragma unroll
      for (int kk = 0; kk < SC_KT; ++kk) {
        float p = coef * fast_exp2(l[kk] - m);
        p += __shfl_xor_sync(0xffffffffu, p, 4);
        p += __shfl_xor_sync(0xffffffffu, p, 2);
        p += __shfl_xor_sync(0xffffffffu, p, 1);
        if (c == 0) sbuf[ql][kk] = p;
      }
      __syncthreads();
      for (int e = tid; e < 16 * SC_KT; e += SC_THREADS) {
        const int r = e / SC_KT, kk = e - r * SC_KT;
        const int q2 = g * 16 + r;
        if (q2 < a.nQ && kk < nk) a.S[((size_t)bh * a.nQ + q2) * a.nK + j0 + kk] = sbuf[r][kk];
      }
    }
  }
  if (PASS == 1 && live) {
    a.stats[crow * 2] = m;
    a.stats[crow * 2 + 1] = z;
  }
}

}  // namespace abattn
