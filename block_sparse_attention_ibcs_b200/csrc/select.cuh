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
// the CPU reference bit for bit.  Assignments are decided in fp32 with a certified error
// margin; a row whose best and second-best distances are closer than that margin is
// decided again in fp64, so the labels equal the exact argmin.  Logits use the bf16
// operands with fp32 accumulation; softmax statistics are fp32 in the log2 domain.
//
//   pool_kernel      Kp[bh, j, :]  = bf16(mean of block j's valid keys)
//   kmeans_kernel    per (bh, query block): centroids (bf16) and shares (fp32)
//   score_kernel<1>  per centroid row and key chunk: reference m and sum z of exp2(logit - m)
//   score_kernel<2>  S[bh, i, j] = sum_c (w_c / Z_c) exp2(logit_cj - m_c)
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
  float* stats;      // [BH, groups of 32 query blocks, 256 rows, 8 key chunks] of (m, z):
                     // reference m (log2 units) and sum z of exp2(logit - m) per chunk
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
    auto add_row = [&](const uint4 v) {
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_to_double((uint16_t)(w4[e] & 0xffffu));
        acc[2 * e + 1] += bf16_to_double((uint16_t)(w4[e] >> 16));
      }
    };
    const int n = t1 - t0;
    if (n == 4) {  // the usual 4-token block: its four row loads in flight together
      uint4 v[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) v[t] = __ldg((const uint4*)(src + t * D));
#pragma unroll
      for (int t = 0; t < 4; ++t) add_row(v[t]);
    } else {
      for (int t = 0; t < n; ++t) add_row(__ldg((const uint4*)(src + t * D)));
    }
    // a power-of-two count divides exactly as a multiplication by its reciprocal
    const double cnt = (double)n, inv = 1.0 / cnt;
    const bool pow2 = (n & (n - 1)) == 0;
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double m0 = pow2 ? acc[2 * e] * inv : acc[2 * e] / cnt;
      const double m1 = pow2 ? acc[2 * e + 1] * inv : acc[2 * e + 1] / cnt;
      o[e] = (uint32_t)bf16_bits_from_double(m0) | ((uint32_t)bf16_bits_from_double(m1) << 16);
    }
    *(uint4*)(a.Kp + bj * D + u * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ k-means
//
// One CTA of 256 threads per (bh, query block).
//  * Segment means (the start) and member means (the update) are exact fp64 sums of the
//    bf16 rows divided by the count (IEEE division; a power-of-two count as the exact
//    multiplication by its reciprocal), as the CPU reference computes them.  Sums of at
//    most 128 bf16 values are exact in fp64, so their order does not matter: the update
//    visits the rows in label order (a counting sort), two or four threads per dimension
//    taking alternate rows of each cluster and adding their partial sums by shuffles.
//  * Assignment: two threads per row compute the 8 squared distances in fp32 against the
//    fp32-rounded centroids as |q|^2 + |c|^2 - 2 q.c (one fma per column and centroid).
//    With u = 2^-24 each fp32 distance is within (d + d/32 + 14) u (|q|^2 + |c|^2) of the
//    exact one: the two d/2-term q.c chains and their sum (doubled), the rounding of c to
//    fp32, the |q|^2 and |c|^2 sums, and the final two roundings (|q.c| is at most half of
//    |q|^2 + |c|^2).  So when the best and second-best fp32 distances are further apart
//    than the best's bound plus the largest bound of any cluster, the fp32 choice is the
//    exact argmin.  Rows inside the margin are recomputed in fp64 (ties to the lowest
//    cluster), like the reference.

template <int D>
__global__ void __launch_bounds__(KM_THREADS) kmeans_kernel(SelectArgs a) {
  __shared__ __align__(16) uint16_t qs[128 * D];
  __shared__ double c64[CMAX * D];
  __shared__ __align__(16) float cf[CMAX * D];
  __shared__ float c2[CMAX];
  __shared__ int cnt[CMAX];
  __shared__ int off[CMAX];
  __shared__ int alive[CMAX];
  __shared__ int sb[CMAX + 1];  // segment c = rows [sb[c], sb[c+1])
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
  if (tid <= CMAX) sb[tid] = (tid <= C) ? tid * n / C : n;  // one division per bound
  __syncthreads();
  if (tid < CMAX) {
    cnt[tid] = (tid < C) ? sb[tid + 1] - sb[tid] : 0;
    alive[tid] = (tid < C) && (sb[tid + 1] > sb[tid]);
  }
  if (tid < 128) {
    int c = -1;
    if (tid < n)
      for (int cc = 0; cc < C; ++cc)
        if (tid >= sb[cc] && tid < sb[cc + 1]) c = cc;
    lab[tid] = (int8_t)c;
  }
  // segment means (fp64, exact sums, so the order of the additions does not matter):
  // thread (segment, dimension pair) loads both dimensions of a row at once and keeps four
  // partial sums per dimension, so the loads and adds of four rows are in flight together
  {
    const uint32_t* qs32 = (const uint32_t*)qs;
    for (int p2 = tid; p2 < CMAX * (D / 2); p2 += KM_THREADS) {
      const int c = p2 / (D / 2), dp = p2 - c * (D / 2);
      double ea[4] = {0.0, 0.0, 0.0, 0.0}, eb[4] = {0.0, 0.0, 0.0, 0.0};  // dimensions 2dp, 2dp + 1
      const int s0 = c < C ? sb[c] : 0, s1 = c < C ? sb[c + 1] : 0;
      int r = s0;
      for (; r + 3 < s1; r += 4) {
        uint32_t wv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) wv[k] = qs32[(r + k) * (D / 2) + dp];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ea[k] += (double)__uint_as_float(wv[k] << 16);
          eb[k] += (double)__uint_as_float(wv[k] & 0xffff0000u);
        }
      }
      for (; r < s1; ++r) {  // the ragged tail (exact sums: any partial will do)
        const uint32_t w = qs32[r * (D / 2) + dp];
        ea[0] += (double)__uint_as_float(w << 16);
        eb[0] += (double)__uint_as_float(w & 0xffff0000u);
      }
      double sa = (ea[0] + ea[1]) + (ea[2] + ea[3]), sbb = (eb[0] + eb[1]) + (eb[2] + eb[3]);
      const int len = s1 - s0;
      if (len > 0) {
        if ((len & (len - 1)) == 0) {
          sa *= 1.0 / (double)len;
          sbb *= 1.0 / (double)len;
        } else {
          sa /= (double)len;
          sbb /= (double)len;
        }
      }
      c64[c * D + 2 * dp] = sa;
      c64[c * D + 2 * dp + 1] = sbb;
    }
  }
  __syncthreads();

  const int ar = tid >> 1;   // assignment: row
  const int ah = tid & 1;    // ... and which half of the dimensions
  for (int it = 0; it < a.iters; ++it) {
    // fp32 copies of the centroids and their squared norms
    for (int p = tid; p < CMAX * D; p += KM_THREADS) cf[p] = (float)c64[p];
    __syncthreads();
    {  // |c|^2: warp c for centroid c (KM_THREADS / 32 = CMAX warps)
      const int c = tid >> 5, l = tid & 31;
      float part = 0.f;
      for (int dd = l; dd < D; dd += 32) part = fmaf(cf[c * D + dd], cf[c * D + dd], part);
#pragma unroll
      for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (l == 0) c2[c] = part;
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
        for (int c = 0; c < CMAX; ++c) {  // dist[c] accumulates q . c here
          const float* cc = cf + c * D + ah * H + e;
          const float4 c0 = *(const float4*)cc;
          const float4 c1 = *(const float4*)(cc + 4);
          const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) dist[c] = fmaf(qv[k], cv[k], dist[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < CMAX; ++c) dist[c] += __shfl_xor_sync(0xffffffffu, dist[c], 1);
      q2 += __shfl_xor_sync(0xffffffffu, q2, 1);
#pragma unroll
      for (int c = 0; c < CMAX; ++c) dist[c] = (q2 + c2[c]) - 2.f * dist[c];  // |q - c|^2
      int best = -1, second = -1;
      float d1 = 0.f, d2 = 0.f, n1 = 0.f, nmax = 0.f;  // best / second distance, |c_best|^2, max |c|^2
#pragma unroll
      for (int c = 0; c < CMAX; ++c) {
        if (!alive[c]) continue;
        nmax = fmaxf(nmax, c2[c]);
        if (best < 0 || dist[c] < d1) {
          second = best; d2 = d1;
          best = c; d1 = dist[c]; n1 = c2[c];
        } else if (second < 0 || dist[c] < d2) {
          second = c; d2 = dist[c];
        }
      }
      constexpr float U = 5.9604645e-8f;  // 2^-24
      bool certain = true;
      if (second >= 0) {
        const float kb = (float)(D + D / 32 + 16) * U * 1.0625f;  // bound factor with margin
        certain = d2 - d1 > kb * ((q2 + n1) + (q2 + nmax));
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
    // update: KM_THREADS / D adjacent threads share a dimension and walk alternate rows of
    // each cluster (label order); their partial sums meet by shuffles
    {
      constexpr int PARTS = KM_THREADS / D;  // 2 at d = 128, 4 at d = 64
      const int dd = tid / PARTS, h = tid % PARTS;
      int r0 = 0;
      for (int c = 0; c < CMAX; ++c) {
        const int k = cnt[c];  // block-uniform
        if (k > 0) {
          double acc0 = 0.0, acc1 = 0.0;  // two partial sums: two members' loads in flight
          int q = r0 + h;
          for (; q + PARTS < r0 + k; q += 2 * PARTS) {
            const int ra = perm[q], rb = perm[q + PARTS];
            acc0 += bf16_to_double(qs[ra * D + dd]);
            acc1 += bf16_to_double(qs[rb * D + dd]);
          }
          if (q < r0 + k) acc0 += bf16_to_double(qs[perm[q] * D + dd]);
          double acc = acc0 + acc1;
#pragma unroll
          for (int o = 1; o < PARTS; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (h == 0) c64[c * D + dd] = acc;  // the member sum; divided below
        }
        r0 += k;
      }
    }
    __syncthreads();
    // member means: the 1024 divisions spread over all threads (independent of each other)
    for (int p = tid; p < CMAX * D; p += KM_THREADS) {
      const int k = cnt[p / D];
      if (k > 0) c64[p] = c64[p] / (double)k;
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
// matrix operations) as two persistent tensor-core streaming passes.  A group is 32 query
// blocks of one head (256 centroid rows); its key axis is cut into at most 8 chunks of
// whole 128-key tiles (the count chosen per shape, see score_split).  The (group, chunk) units, numbered head by head, are dealt out
// round-robin to one CTA per SM, so the CTAs running at any moment work on about one
// head and share its pooled keys in L2 (all heads' pooled keys together exceed L2 at the
// Wan2.1-14B shape).  A CTA loads a unit's centroids, then streams the chunk's key tiles;
// the first key tiles of the next unit are requested before its centroids, so the
// centroid reload overlaps the end of the previous unit.
//   PASS 1: D[centroid row, key] = C Kp^T for the two 128-row halves of the centroids
//           (A = centroids, B = key tile, both K-major, N = 128).  Each thread keeps a
//           running reference m and sum z of exp2(logit - m) for one centroid row over
//           the unit's keys.  m is raised lazily: a 32-key chunk whose sum stays
//           below 2^20 is accepted as it is (a term can then exceed 1 by at most 2^20,
//           far from fp32 overflow); otherwise the chunk's maximum is taken and z rescaled.
//           At the end of each unit the two groups' (m, z) of a row are merged and stored
//           in the slot of the unit's key chunk; pass 2 merges a row's slots in chunk order, so S does not depend on how
//           the units were dealt out to CTAs.
//   PASS 2: D[key, centroid column] = Kp C^T (A = key tile, B = all 256 centroid rows,
//           N = 256), so thread j owns one KV block and sums exp2(logit - m'_c) over the
//           8 columns of each of its 16 query blocks in registers, where the share and
//           the softmax normaliser are folded into one constant per column:
//           w_c exp2(l - m_c) / Z_c = exp2(l - (m_c + log2 Z_c - log2 w_c)).
//           S rows are stored coalesced.
// Roles: warps 0-15 consume TMEM in two groups that alternate tiles (group g = warp / 8
// takes the unit's tiles t0 + g, t0 + g + 2, ..., which the MMAs put in TMEM buffer g), so one group's exponentials cover the other's TMEM
// loads; in a group, lane quadrant = warp % 4 and each thread reads 128 columns of its
// tile in four 32-column chunks.  One thread of warp 16 streams the centroids and the key tiles with TMA (3-D
// tiled boxes with the 128-byte swizzle the MMA descriptors expect; rows past the head's
// end are filled with zeros), 3 stages deep; warp 17 allocates 512 TMEM columns and one of
// its threads issues the MMAs.

constexpr int SC_QB = 32;                  // query blocks per group
constexpr int SC_ROWS = SC_QB * CMAX;      // 256 centroid rows per group
constexpr int SC_CONSUMERS = 512;          // warps 0-15: two groups of 8
constexpr int SC_GROUP = 256;              // consumers of one TMEM buffer
constexpr int SC_PRODUCER_WARP = 16;       // TMA producer
constexpr int SC_MMA_WARP = 17;            // TMEM allocation, MMA issue
constexpr int SC_THREADS = SC_CONSUMERS + 64;
constexpr int SC_STAGES = 3;
constexpr int SC_MAX_CHUNKS = 8;           // key chunks per group (pass-1 partial slots)
// The chunk count is chosen for a fixed nominal grid of 148 CTAs (B200's SM count), not
// for the device at hand: chunk boundaries decide how S is rounded, so S stays the same
// on every device.  The launch itself uses one CTA per SM of the device.
constexpr int SC_SPLIT_GRID = 148;
constexpr float SC_LAZY_LIMIT = 1048576.f;  // 2^20

template <int D>
struct ScoreSmem {
  static constexpr uint32_t CCHUNK = SC_ROWS * 128u;  // one 64-element column chunk, 256 rows
  static constexpr uint32_t CENT_BYTES = (D / 64) * CCHUNK;
  static constexpr uint32_t KCHUNK = 128u * 128u;
  static constexpr uint32_t KTILE = (D / 64) * KCHUNK;
  static constexpr uint32_t CENT_OFF = 0;
  static constexpr uint32_t KP_OFF = CENT_OFF + CENT_BYTES;
  static constexpr uint32_t COL_OFF = KP_OFF + SC_STAGES * KTILE;  // pass 2: m' per column
  static constexpr uint32_t MERGE_OFF = COL_OFF + SC_ROWS * 4u;      // pass 1: (m, z) per row
  static constexpr uint32_t BAR_OFF = MERGE_OFF + SC_ROWS * 8u;
  // CFULL, CEMPTY, FULL[3], EMPTY[3], SFULL[2], SFREE[2], DRAIN
  static constexpr uint32_t NBARS = 13;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBARS * 8u;
  static constexpr uint32_t BYTES = MISC_OFF + 16u;
  static constexpr uint32_t ALLOC = BYTES + 1024u;
  static_assert(KP_OFF % 1024u == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(ALLOC <= 232448u, "exceeds the 227 KB shared-memory limit per block");
};

enum { SB_CFULL = 0, SB_CEMPTY = 1, SB_FULL0 = 2, SB_EMPTY0 = 5, SB_SFULL0 = 8, SB_SFREE0 = 10,
       SB_DRAIN = 12 };

// The work split shared by both passes (host and device compute it the same way).
struct ScoreSplit {
  int G;        // groups per head: ceil(nQ / 32)
  int T;        // 128-key tiles per row: ceil(nK / 128)
  int CT;       // tiles per chunk
  int KC;       // chunks per group: ceil(T / CT) <= SC_MAX_CHUNKS
  long long U;  // units = B*H * G * KC
  int P;        // CTAs = min(U, SMs of the device)
};

// The number of key chunks per group trades load balance (more, shorter units) against
// the centroid reload at every unit (measured on B200 at about two tiles of time): choose
// the count that minimises (units of the busiest CTA) x (tiles per unit + 2) for a tensor
// of BH_choice heads on the nominal grid.  A launch over a slice of heads passes the whole
// layer's head count, so its chunks -- and with them the rounding of S -- are those of one
// launch over the whole layer.
inline ScoreSplit score_split(long long BH, long long nQ, long long nK, long long BH_choice,
                              int sms) {
  ScoreSplit s;
  s.G = (int)((nQ + SC_QB - 1) / SC_QB);
  s.T = (int)((nK + 127) / 128);
  const long long R = BH_choice * s.G;
  long long best = -1;
  for (int k = 1; k <= SC_MAX_CHUNKS && k <= s.T; ++k) {
    const int ct = (s.T + k - 1) / k;
    const int kc = (s.T + ct - 1) / ct;
    const long long per_cta = (R * kc + SC_SPLIT_GRID - 1) / SC_SPLIT_GRID;
    const long long cost = per_cta * (ct + 2);
    if (best < 0 || cost < best) {
      best = cost;
      s.CT = ct;
      s.KC = kc;
    }
  }
  s.U = BH * s.G * s.KC;
  s.P = (int)(s.U < sms ? s.U : sms);
  return s;
}

// Exponentials per 32-logit chunk (pass 1) and per 8-column query block (pass 2) that go
// to the FMA-pipe polynomial instead of the MUFU, in pairs: of 16 and of 4 pairs.
#ifndef SC_POLY_PAIRS1
#define SC_POLY_PAIRS1 2
#endif
#ifndef SC_POLY_PAIRS2
#define SC_POLY_PAIRS2 0
#endif

// Sum over 32 logits of exp2(l * c + nm), in packed pairs; the first NP of the 16 pairs use
// the polynomial exp2, the others the MUFU.  Four independent partial sums.
template <int NP>
AB_DEV float expsum32(const uint32_t (&v)[32], float c, float nm) {
  const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(nm, nm);
  uint64_t a[4] = {0, 0, 0, 0};  // (0.f, 0.f)
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), c2, nm2));
    const uint64_t e = (i < NP) ? exp2_poly_x2(x.x, x.y) : f2_pack(fast_exp2(x.x), fast_exp2(x.y));
    a[i & 3] = f2_add(a[i & 3], e);
  }
  const float2 s = f2_unpack(f2_add(f2_add(a[0], a[1]), f2_add(a[2], a[3])));
  return s.x + s.y;
}

// Adds a chunk of 32 logits to the running (m, z) of one centroid row (see PASS 1 above).
AB_DEV void online_chunk(const uint32_t (&v)[32], float c, float& m, float& z) {
  float acc = expsum32<SC_POLY_PAIRS1>(v, c, -m);
  if (m == -INFINITY || !(acc <= SC_LAZY_LIMIT)) {  // first chunk, a maximum far above m, or NaN
    float mt = -INFINITY;
#pragma unroll
    for (int k = 0; k < 32; ++k) mt = fmaxf(mt, __uint_as_float(v[k]));
    const float mn = fmaxf(m, mt * c);
    if (mn == -INFINITY) {
      acc = 0.f;  // every key is masked
    } else {
      z = (m == -INFINITY) ? 0.f : z * fast_exp2(m - mn);
      m = mn;
      acc = expsum32<0>(v, c, -m);
    }
  }
  z += acc;
}

template <int D, int PASS>
__global__ void __launch_bounds__(SC_THREADS, 1) score_kernel(
    SelectArgs a, ScoreSplit sp, const __grid_constant__ CUtensorMap tm_kp,
    const __grid_constant__ CUtensorMap tm_cent, uint64_t timeout_ns) {
  using L = ScoreSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF);
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF + 4);
  float* col_m = (float*)(smem + L::COL_OFF);
  float2* merge = (float2*)(smem + L::MERGE_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars[SB_CFULL], 1);
    mbar_init(&bars[SB_CEMPTY], 1);
    for (int b = 0; b < SC_STAGES; ++b) {
      mbar_init(&bars[SB_FULL0 + b], 1);
      mbar_init(&bars[SB_EMPTY0 + b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[SB_SFULL0 + b], 1);
      mbar_init(&bars[SB_SFREE0 + b], SC_GROUP);
    }
    mbar_init(&bars[SB_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == SC_MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Units of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...  Unit un is chunk
  // k = un % KC of group gi = un / KC: tiles [k * CT, min(T, (k + 1) * CT)).
  auto unit = [&](long long un, long long& gi, int& t0, int& t1) {
    gi = un / sp.KC;
    const int k = (int)(un - gi * sp.KC);
    t0 = k * sp.CT;
    t1 = min(sp.T, t0 + sp.CT);
  };

  if (warp == SC_PRODUCER_WARP) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      long long it = 0;  // tiles of this CTA so far
      int sg = 0;        // units so far
      bool ok = true;
      auto load_tile = [&](int bh, int t) -> bool {
        const int st = (int)(it % SC_STAGES);
        if (it >= SC_STAGES &&
            !mbar_wait(&bars[SB_EMPTY0 + st], (int)((it / SC_STAGES - 1) & 1), abort_flag, timeout_ns))
          return false;
        mbar_arrive_expect_tx(&bars[SB_FULL0 + st], L::KTILE);
#pragma unroll
        for (int ck = 0; ck < D / 64; ++ck)  // keys t*128 .. t*128 + 127 of head bh
          tma_load_3d(sbase + L::KP_OFF + st * L::KTILE + ck * L::KCHUNK, &tm_kp, ck * 64, t * 128, bh,
                      &bars[SB_FULL0 + st]);
        ++it;
        return true;
      };
      for (long long un = blockIdx.x; un < sp.U && ok; un += gridDim.x, ++sg) {
        long long gi;
        int t0, t1;
        unit(un, gi, t0, t1);
        const int bh = (int)(gi / sp.G);
        const int qb0 = (int)(gi - (long long)bh * sp.G) * SC_QB;
        int t = t0;
        if (sg > 0) {  // the first key tiles, then wait until the centroid buffer is free
          for (; t < min(t1, t0 + SC_STAGES) && ok; ++t) ok = load_tile(bh, t);
          if (!ok || !mbar_wait(&bars[SB_CEMPTY], (sg - 1) & 1, abort_flag, timeout_ns)) {
            ok = false;
            break;
          }
        }
        mbar_arrive_expect_tx(&bars[SB_CFULL], L::CENT_BYTES);
#pragma unroll
        for (int ck = 0; ck < D / 64; ++ck)  // centroid rows qb0*8 .. qb0*8 + 255 of head bh
          tma_load_3d(sbase + L::CENT_OFF + ck * L::CCHUNK, &tm_cent, ck * 64, qb0 * CMAX, bh, &bars[SB_CFULL]);
        for (; t < t1 && ok; ++t) ok = load_tile(bh, t);
      }
      // let copies still in flight land before the CTA can exit (only after an abort)
      for (long long k = (it > SC_STAGES ? it - SC_STAGES : 0); k < it; ++k)
        mbar_wait_quiet(&bars[SB_FULL0 + (int)(k % SC_STAGES)], (int)((k / SC_STAGES) & 1), timeout_ns);
      if (sg > 0) mbar_wait_quiet(&bars[SB_CFULL], (sg - 1) & 1, timeout_ns);  // sg centroid loads issued
    }
    __syncwarp();
  } else if (warp == SC_MMA_WARP) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC1 = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC2 = idesc_bf16_f32(128, SC_ROWS, 0, 0);
      long long it = 0;
      int sg = 0;
      int nuse[2] = {0, 0};  // tiles issued into each TMEM buffer
      bool ok = true;
      for (long long un = blockIdx.x; un < sp.U && ok; un += gridDim.x, ++sg) {
        long long gi;
        int t0, t1;
        unit(un, gi, t0, t1);
        if (!(ok = mbar_wait(&bars[SB_CFULL], sg & 1, abort_flag, timeout_ns))) break;
        for (int t = t0; t < t1; ++t, ++it) {
          const int st = (int)(it % SC_STAGES), b = (t - t0) & 1;
          ok = mbar_wait(&bars[SB_FULL0 + st], (int)((it / SC_STAGES) & 1), abort_flag, timeout_ns);
          if (ok && nuse[b] > 0) ok = mbar_wait(&bars[SB_SFREE0 + b], (nuse[b] - 1) & 1, abort_flag, timeout_ns);
          if (!ok) break;
          ++nuse[b];
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t cbase = sbase + L::CENT_OFF;
          const uint32_t kbase = sbase + L::KP_OFF + st * L::KTILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk & 3) * 32;
            const uint64_t dk = sdesc_sw128(kbase + (kk >> 2) * L::KCHUNK + ko, 16, 1024);
            const uint64_t dc = sdesc_sw128(cbase + (kk >> 2) * L::CCHUNK + ko, 16, 1024);
            if (PASS == 1) {
              umma_f16_ss(tmem + b * 256, dc, dk, IDESC1, kk > 0 ? 1u : 0u);
              const uint64_t dc1 = sdesc_sw128(cbase + (kk >> 2) * L::CCHUNK + 128u * 128u + ko, 16, 1024);
              umma_f16_ss(tmem + b * 256 + 128, dc1, dk, IDESC1, kk > 0 ? 1u : 0u);
            } else {
              umma_f16_ss(tmem + b * 256, dk, dc, IDESC2, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&bars[SB_SFULL0 + b]);
          umma_commit(&bars[SB_EMPTY0 + st]);
        }
        umma_commit(&bars[SB_CEMPTY]);  // the centroid buffer is free once these MMAs end
      }
      umma_commit(&bars[SB_DRAIN]);
      mbar_wait(&bars[SB_DRAIN], 0, abort_flag, timeout_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers (warps 0-15)
    const int q = warp & 3, sub = (warp >> 2) & 1, grp = warp >> 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float c = a.scale_log2;
    int nuse = 0;  // tiles of this group's TMEM buffer so far
    bool ok = true;
    for (long long un = blockIdx.x; un < sp.U; un += gridDim.x) {
      long long gi;
      int t0, t1;
      unit(un, gi, t0, t1);
      const long long bh = gi / sp.G;
      const int qb0 = (int)(gi - bh * sp.G) * SC_QB;
      if (PASS == 2) {
        // the column constants m' of this group (every consumer passes both barriers)
        asm volatile("bar.sync 1, %0;" ::"n"(SC_CONSUMERS) : "memory");
        if (tid < SC_ROWS) {
          const int qb = qb0 + (tid >> 3);
          float mp = INFINITY;
          if (qb < a.nQ) {
            const float2* sl = (const float2*)a.stats + ((size_t)gi * SC_ROWS + tid) * SC_MAX_CHUNKS;
            float M = -INFINITY, Z = 0.f;
            for (int k = 0; k < sp.KC; ++k) M = fmaxf(M, sl[k].x);
            if (M > -INFINITY)
              for (int k = 0; k < sp.KC; ++k) {
                const float2 mz = sl[k];
                if (mz.x > -INFINITY) Z += mz.y * fast_exp2(mz.x - M);
              }
            const float w = a.w[((size_t)bh * a.nQ + qb) * CMAX + (tid & 7)];
            if (w > 0.f && Z > 0.f && M > -INFINITY) mp = M + (log2f(Z) - log2f(w));
          }
          col_m[tid] = mp;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(SC_CONSUMERS) : "memory");
      }
      // pass 1: row sub * 128 + 32 q + lane (centroid half sub); pass 2: key 32 q + lane of the
      // tile and centroid columns sub * 128 .. + 127 (query blocks sub * 16 .. + 15)
      const uint32_t cols = (uint32_t)(sub * 128);
      float m = -INFINITY, z = 0.f;
      auto compute = [&](uint32_t (&v)[32], int t, int part) {
        if (PASS == 1) {
          const int jb = t * 128 + part * 32;  // key of v[0]
          if (jb + 32 > a.nK) {                // the ragged last tile: mask keys >= nK
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (jb + e >= a.nK) v[e] = __float_as_uint(-INFINITY);
          }
          online_chunk(v, c, m, z);
        } else {
          const int j = t * 128 + q * 32 + lane;
          const uint64_t c2 = f2_pack(c, c);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int cb = sub * 128 + part * 32 + qq * 8;  // first column of this query block
            float mp[8];
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(mp[0]), "=f"(mp[1]), "=f"(mp[2]), "=f"(mp[3])
                         : "r"(smem_u32(col_m + cb)));
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(mp[4]), "=f"(mp[5]), "=f"(mp[6]), "=f"(mp[7])
                         : "r"(smem_u32(col_m + cb + 4)));
            uint64_t acc = 0;  // (0.f, 0.f)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(v[qq * 8 + 2 * e]),
                                                        __uint_as_float(v[qq * 8 + 2 * e + 1])),
                                                c2, f2_pack(-mp[2 * e], -mp[2 * e + 1])));
              acc = f2_add(acc, (e < SC_POLY_PAIRS2) ? exp2_poly_x2(x.x, x.y)
                                                    : f2_pack(fast_exp2(x.x), fast_exp2(x.y)));
            }
            const float2 sv = f2_unpack(acc);
            const int qb = qb0 + (cb >> 3);
            if (j < a.nK && qb < a.nQ) a.S[((size_t)bh * a.nQ + qb) * a.nK + j] = sv.x + sv.y;
          }
        }
      };
      // this group's tiles of the unit: t - t0 = grp, grp + 2, ... (they are in TMEM buffer
      // grp), so the split, and with it the rounding of (m, z), depends only on the unit
      for (int t = t0 + grp; t < t1; t += 2) {
        if (ok) ok = mbar_wait(&bars[SB_SFULL0 + grp], nuse & 1, abort_flag, timeout_ns);
        ++nuse;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) continue;
        tc_fence_after();
        const uint32_t base = tmem + lane_off + (uint32_t)(grp * 256) + cols;
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(base + part * 32, v);
          tmem_wait_ld_regs(v);
          if (part == 3) {  // the group has read its whole tile: the buffer is free
            tc_fence_before();
            mbar_arrive(&bars[SB_SFREE0 + grp]);
          }
          compute(v, t, part);
        }
      }
      if (PASS == 1) {
        // merge the two groups' (m, z) of each row and store the unit's slot.  Each chunk's
        // (m, z) depends only on its own keys, so S does not depend on how the units were
        // dealt out to CTAs.
        asm volatile("bar.sync 1, %0;" ::"n"(SC_CONSUMERS) : "memory");
        const int row = sub * 128 + q * 32 + lane;
        if (grp == 1) merge[row] = make_float2(m, z);
        asm volatile("bar.sync 1, %0;" ::"n"(SC_CONSUMERS) : "memory");
        if (grp == 0 && ok) {
          const float2 o = merge[row];
          const float M = fmaxf(m, o.x);
          float Z = 0.f;
          if (M > -INFINITY) {
            if (m > -INFINITY) Z += z * fast_exp2(m - M);
            if (o.x > -INFINITY) Z += o.y * fast_exp2(o.x - M);
          }
          ((float2*)a.stats)[((size_t)gi * SC_ROWS + row) * SC_MAX_CHUNKS + t0 / sp.CT] = make_float2(M, Z);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == SC_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace abattn
