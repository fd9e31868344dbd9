// Packed-tile sparse attention for sm_100a (tcgen05 + TMEM + cp.async gather).
//
// AB-Attention page (onedev.kr/papers/1521), section "premises & limits": the kernel
// gathers the sampled small KV blocks by index into full tensor-core tiles and does
// the inverse-inclusion-probability logit shift, online softmax and value
// accumulation in one attention pass, without reordering tokens; section "how to
// use": weighting a sampled block by 1/pi equals shifting its logits by -log pi.
//
// One CTA per (b, h, query block of 128 rows).  The s sampled blocks (ascending) are
// laid end to end and cut into T = ceil(s*bk/128) tiles of 128 tokens; tile t holds
// tokens t*128 .. t*128+127 of that sequence.  Roles (288 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Reads S from TMEM,
//              adds the shift, lazy online softmax (the running max is only raised
//              when a tile exceeds it by more than 2^8), writes P (bf16) to shared
//              memory, rescales its O row in TMEM when the max moved, and finally
//              writes O / l.
//   warps 4-7  producers: cp.async gather of the tile's K and V rows into 128B-swizzled
//              tiles (two stages) plus the per-column shift; zero rows for padding.
//   warp  8    TMEM allocation; lane 0 issues the MMAs:
//              S[t%2] = Q K_t^T  (M=128, N=128, K=d; both operands K-major)
//              O     += P_t V_t  (M=128, N=d,  K=128; V read MN-major)
// All waits are bounded (mbar_wait); a stuck pipeline records AB_ERR_DEVICE_TIMEOUT and
// every role drains and exits.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int ATTN_THREADS = 288;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;

struct AttnArgs {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;    // [BH, nQ, s] (packed mode)
  const float* logpi;    // [BH, nQ, s]
  uint16_t* O;
  int N, nQ, nK, s, bk, bk_shift;
  int ntiles;            // tiles per query block
  float scale_log2;      // log2(e) / sqrt(d)
  uint64_t timeout_ns;
  int debug_skip_arrive; // test knob: producers skip the first tile's arrival
};

template <int D>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = 128u * D * 2u;  // 128 rows x D bf16
  static constexpr uint32_t CHUNK_BYTES = 128u * 128u;   // one 64-column chunk of 128 rows
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE_BYTES;        // 2 stages
  static constexpr uint32_t V_OFF = K_OFF + 2 * TILE_BYTES;    // 2 stages
  static constexpr uint32_t P_BYTES = 128u * 128u * 2u;       // 128 x 128 bf16
  static constexpr uint32_t P_OFF = V_OFF + 2 * TILE_BYTES;    // 2 buffers
  static constexpr uint32_t BIAS_OFF = P_OFF + 2 * P_BYTES;    // 2 x 128 fp32
  static constexpr uint32_t BAR_OFF = BIAS_OFF + 2u * 128u * 4u;
  static constexpr uint32_t NBARS = 14;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBARS * 8u;
  static constexpr uint32_t BYTES = MISC_OFF + 16u;
  static constexpr uint32_t ALLOC = BYTES + 1024u;  // slack for 1024-byte alignment
  static_assert(ALLOC <= 232448u, "exceeds the 227 KB shared-memory limit per block");
};

// barrier slots (pairs are indexed by tile parity)
enum { B_QFULL = 0, B_FULL0 = 1, B_EMPTY0 = 3, B_SFULL0 = 5, B_SFREE0 = 7, B_PFULL0 = 9,
       B_PVDONE0 = 11, B_DRAIN = 13 };

template <int D, bool DENSE>
__global__ void __launch_bounds__(ATTN_THREADS, 1) attn_kernel(AttnArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  float* bias = (float*)(smem + L::BIAS_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF);
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bh = blockIdx.x / a.nQ;
  const int qb = blockIdx.x - bh * a.nQ;
  const int T = a.ntiles;
  const size_t head_off = (size_t)bh * a.N * D;
  const int row0 = qb * 128;
  const int nvalid = min(128, a.N - row0);

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars[B_QFULL], 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_FULL0 + b], 256);  // 128 plain arrivals + 128 cp.async arrivals
      mbar_init(&bars[B_EMPTY0 + b], 1);
      mbar_init(&bars[B_SFULL0 + b], 1);
      mbar_init(&bars[B_SFREE0 + b], 128);
      mbar_init(&bars[B_PFULL0 + b], 128);
      mbar_init(&bars[B_PVDONE0 + b], 1);
    }
    mbar_init(&bars[B_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t TM_S0 = tmem;        // columns [0,128)
  const uint32_t TM_S1 = tmem + 128;  // columns [128,256)
  const uint32_t TM_O = tmem + 256;   // columns [256, 256+D)

  if (warp >= 4 && warp < 8) {
    // ================================================================ producers
    const int p = tid - 128;       // 0..127
    const int u = p & 15;          // 16-byte unit within a 256-byte (D=128) row
    const int rsub = p >> 4;       // 0..7: this thread copies rows rsub, rsub+8, ...
    constexpr int UNITS = D / 8;   // 16-byte units per row
    const size_t plan_off = (size_t)blockIdx.x * a.s;
    const int nb = 128 >> a.bk_shift;  // sampled blocks per tile

    // Plan entries of one tile, spread over the warp: lane e (+32k) holds the tile's
    // block e -- its index (-1 for padding or a rejected entry) and log pi.  Loaded
    // coalesced one tile ahead and broadcast to the copying lanes with shuffles.
    int jc[4], jn[4];
    float lc[4], ln[4];
    auto fetch = [&](int t, int (&jr)[4], float (&lr)[4]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = lane + 32 * k;
        const int m = t * nb + e;
        jr[k] = -1;
        lr[k] = 0.f;
        if (!DENSE && e < nb && m < a.s) {
          const int j = __ldg(a.idx + plan_off + m);
          if (j < 0 || j >= a.nK) {
            ab_flag(AB_ERR_DEVICE_CHECK);
          } else {
            jr[k] = j;
            lr[k] = __ldg(a.logpi + plan_off + m);
          }
        }
      }
    };
    if (!DENSE) fetch(0, jc, lc);

    // Q tile: rows row0..row0+127 (zero beyond N)
    for (int r = rsub; r < 128; r += 8) {
      if (u < UNITS) {
        const bool ok = r < nvalid;
        const uint16_t* src = a.Q + head_off + (size_t)(ok ? row0 + r : 0) * D + u * 8;
        const uint32_t dst = sbase + L::Q_OFF + (u >> 3) * L::CHUNK_BYTES + sw128_off(r, u & 7);
        cp_async_16(dst, src, ok ? 16u : 0u);
      }
    }
    mbar_arrive_cpasync(&bars[B_QFULL]);

    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (!DENSE && t + 1 < T) fetch(t + 1, jn, ln);  // in flight while this tile is issued
      if (t >= 2 && !mbar_wait(&bars[B_EMPTY0 + st], ((t >> 1) - 1) & 1, abort_flag, a.timeout_ns))
        break;
      const uint32_t kdst = sbase + L::K_OFF + st * L::TILE_BYTES;
      const uint32_t vdst = sbase + L::V_OFF + st * L::TILE_BYTES;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int r = rsub + 8 * i;  // row of the tile (= column of S)
        int tok;
        float b2;
        bool ok;
        if (DENSE) {
          tok = t * 128 + r;
          ok = tok < a.N;
          b2 = 0.f;
        } else {
          const int ml = r >> a.bk_shift;  // block of the tile holding this row
          const int src = ml & 31;
          int j = __shfl_sync(0xffffffffu, jc[0], src);
          float lp = __shfl_sync(0xffffffffu, lc[0], src);
          if (nb > 32) {  // warp-uniform: more than 32 blocks per tile (kv_block < 4)
            const int reg = ml >> 5;
#pragma unroll
            for (int k = 1; k < 4; ++k) {
              const int jk = __shfl_sync(0xffffffffu, jc[k], src);
              const float lk = __shfl_sync(0xffffffffu, lc[k], src);
              if (reg == k) { j = jk; lp = lk; }
            }
          }
          tok = j * a.bk + (r & (a.bk - 1));
          ok = j >= 0 && tok < a.N;
          b2 = -lp * LOG2E;
        }
        if (u < UNITS) {
          const size_t goff = head_off + (size_t)(ok ? tok : 0) * D + u * 8;
          const uint32_t soff = (u >> 3) * L::CHUNK_BYTES + sw128_off(r, u & 7);
          cp_async_16(kdst + soff, a.K + goff, ok ? 16u : 0u);
          cp_async_16(vdst + soff, a.V + goff, ok ? 16u : 0u);
        }
        if (u == 0) bias[st * 128 + r] = ok ? b2 : -INFINITY;
      }
      if (!DENSE) {
#pragma unroll
        for (int k = 0; k < 4; ++k) { jc[k] = jn[k]; lc[k] = ln[k]; }
      }
      if (a.debug_skip_arrive && t == 0) continue;  // test knob: never signal tile 0
      mbar_arrive(&bars[B_FULL0 + st]);
      mbar_arrive_cpasync(&bars[B_FULL0 + st]);
    }
    cp_async_wait_all();
  } else if (warp == 8) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      bool ok = mbar_wait(&bars[B_QFULL], 0, abort_flag, a.timeout_ns);
      // issue PV for tile tp (P ready, V in stage tp&1)
      auto issue_pv = [&](int tp) -> bool {
        if (!mbar_wait(&bars[B_PFULL0 + (tp & 1)], (tp >> 1) & 1, abort_flag, a.timeout_ns))
          return false;
        tc_fence_after();
        const uint32_t vbase = sbase + L::V_OFF + (tp & 1) * L::TILE_BYTES;
        const uint32_t pbase = sbase + L::P_OFF + (tp & 1) * L::P_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys per MMA
          const uint64_t ad = sdesc_sw128(pbase + (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(vbase + kk * 2048, L::CHUNK_BYTES, 1024);
          umma_f16_ss(TM_O, ad, bd, IDESC_PV, (tp > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_PVDONE0 + (tp & 1)]);
        umma_commit(&bars[B_EMPTY0 + (tp & 1)]);
        return true;
      };
      for (int t = 0; t < T && ok; ++t) {
        const int st = t & 1;
        ok = mbar_wait(&bars[B_FULL0 + st], (t >> 1) & 1, abort_flag, a.timeout_ns);
        if (!ok) break;
        if (t >= 2) {
          ok = mbar_wait(&bars[B_SFREE0 + st], ((t >> 1) - 1) & 1, abort_flag, a.timeout_ns);
          if (!ok) break;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t kbase = sbase + L::K_OFF + st * L::TILE_BYTES;
        const uint32_t qbase = sbase + L::Q_OFF;
        const uint32_t dS = st ? TM_S1 : TM_S0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32;
          umma_f16_ss(dS, sdesc_sw128(qbase + koff, 16, 1024), sdesc_sw128(kbase + koff, 16, 1024),
                      IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_SFULL0 + st]);
        if (t >= 1) ok = issue_pv(t - 1);
      }
      if (ok && T > 0) ok = issue_pv(T - 1);
      // drain: wait until every MMA issued above has completed before TMEM is freed
      umma_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0, abort_flag, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax (warps 0-3)
    const int r = tid;  // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY;  // reference max (log2 domain)
    float l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      // S(t) ready; FULL(t) is waited too, for acquire ordering of the producers' shifts
      ok = mbar_wait(&bars[B_SFULL0 + st], (t >> 1) & 1, abort_flag, a.timeout_ns) &&
           mbar_wait(&bars[B_FULL0 + st], (t >> 1) & 1, abort_flag, a.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const float* bcol = bias + st * 128;
      const uint32_t sadr = (st ? TM_S1 : TM_S0) + lane_off;
      float z[128];
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(sadr + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 b4 = *(const float4*)(bcol + c0 + c);
          z[c0 + c] = fmaf(__uint_as_float(v[c]), a.scale_log2, b4.x);
          z[c0 + c + 1] = fmaf(__uint_as_float(v[c + 1]), a.scale_log2, b4.y);
          z[c0 + c + 2] = fmaf(__uint_as_float(v[c + 2]), a.scale_log2, b4.z);
          z[c0 + c + 3] = fmaf(__uint_as_float(v[c + 3]), a.scale_log2, b4.w);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[B_SFREE0 + st]);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mt = fmaxf(mt, z[c]);
      // Lazy rescale, decided per warp: tcgen05.ld/st are warp-collective, so when any
      // row of the warp has to raise its reference max, every row of the warp moves to
      // max(m_run, mt) (alpha = 1 where nothing changes) and the warp rescales O.
      const bool need = mt > m_run + LAZY_RESCALE_LOG2;  // always true on a row's first finite tile
      const bool rescale = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (rescale) {
        const float m_new = fmaxf(mt, m_run);
        if (m_new != -INFINITY) {
          alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
          m_run = m_new;
        }
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      // P buffer st is free once PV(t-2) has completed
      if (t >= 2) {
        ok = mbar_wait(&bars[B_PVDONE0 + st], ((t >> 1) - 1) & 1, abort_flag, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      uint8_t* prow = smem + L::P_OFF + st * L::P_BYTES;
      float lsum = 0.f;
#pragma unroll
      for (int uu = 0; uu < 16; ++uu) {  // 8 keys per 16-byte unit of P
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = fast_exp2(z[8 * uu + 2 * e] - mref);
          const float p1 = fast_exp2(z[8 * uu + 2 * e + 1] - mref);
          lsum += p0 + p1;
          pk[e] = pack_bf16x2_rn(p0, p1);
        }
        const uint32_t off = (uu >> 3) * 16384u + sw128_off(r, uu & 7);
        *(uint4*)(prow + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l_run = l_run * alpha + lsum;
      if (rescale && t > 0) {  // warp-uniform; O holds no data before PV(0)
        // O is stable once PV(t-1) has completed
        ok = mbar_wait(&bars[B_PVDONE0 + (st ^ 1)], ((t - 1) >> 1) & 1, abort_flag, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(TM_O + lane_off + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * alpha);
          tmem_st_32x32b_x32(TM_O + lane_off + c0, v);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL0 + st]);
    }
    if (ok && T > 0)
      ok = mbar_wait(&bars[B_PVDONE0 + ((T - 1) & 1)], ((T - 1) >> 1) & 1, abort_flag, a.timeout_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      uint16_t* orow = a.O + head_off + (size_t)(row0 + r) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(TM_O + lane_off + c0, v);
        tmem_wait_ld();
        if (r < nvalid) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 o;
            o.x = pack_bf16x2_rn(__uint_as_float(v[c]) * inv, __uint_as_float(v[c + 1]) * inv);
            o.y = pack_bf16x2_rn(__uint_as_float(v[c + 2]) * inv, __uint_as_float(v[c + 3]) * inv);
            o.z = pack_bf16x2_rn(__uint_as_float(v[c + 4]) * inv, __uint_as_float(v[c + 5]) * inv);
            o.w = pack_bf16x2_rn(__uint_as_float(v[c + 6]) * inv, __uint_as_float(v[c + 7]) * inv);
            *(uint4*)(orow + c0 + c) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace abattn
