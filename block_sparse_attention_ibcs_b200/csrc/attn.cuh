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
//   warps 4-7  producers: the Q tile once, then each tile's K rows and then its V rows by
//              16-byte cp.async into 128B-swizzled tiles, three stages deep (a stage is
//              freed when PV of its tile completes); zero rows for padding.  K and V land
//              on separate barriers so QK can start before V has arrived.  The gather of
//              small blocks from L2 bounds this kernel, so every producer warp copies both
//              K and V and the ring is as deep as shared memory allows.
//   warp  8    allocates 512 TMEM columns; lane 0 issues the MMAs, whichever is ready:
//              S[t%2] = Q K_t^T  (M=128, N=128, K=d; A and B from shared memory)
//              O     += P_t V_t  (M=128, N=d,  K=128; A = P from tensor memory, B = V
//                                 read MN-major from the same tile layout)
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Computes column r's
//              shift -log(pi) * log2(e) (-inf for padding) from its prefetched plan entry,
//              reads S from TMEM, adds the shifts, keeps a lazy online max (raised only
//              when a tile exceeds it by more than 2^8, decided per warp), writes P as
//              bf16 into tensor memory, rescales its O row when the max moved, and
//              finally writes O / l.
// Tensor memory: S0 [0,128), S1 [128,256), O [256,256+d), P0 [384,448), P1 [448,512).
// All waits are bounded; a stuck pipeline records AB_ERR_DEVICE_TIMEOUT and every role
// drains and exits.
#pragma once

#include <climits>

#include "common.cuh"

namespace abattn {

constexpr int ATTN_THREADS = 288;
constexpr int ATTN_STAGES = 3;
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
  uint64_t* trace;       // TRACE builds: clock64 per (traced CTA, event, tile)
};

// Event tracing (TRACE builds only): CTAs 0, 1 and the one at a third of the grid record
// clock64() per tile for the events below into trace[((slot * 16) + event) * 128 + t].
enum { EV_COPY_START = 0, EV_COPY_ISSUED, EV_SM_LOADED, EV_SM_MAX, EV_LANDED, EV_QK,
       EV_SM_PBUF, EV_PV, EV_SM_START, EV_SM_READY, EV_SM_PDONE, EV_END, EV_SM_SFULL,
       EV_SM_PDONE_W1, EV_SM_PDONE_W2, EV_SM_PDONE_W3, EV_COUNT };
constexpr int TRACE_TILES = 128;

template <int D>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = 128u * D * 2u;  // 128 rows x D bf16
  static constexpr uint32_t CHUNK_BYTES = 128u * 128u;   // one 64-column chunk of 128 rows
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE_BYTES;                  // ATTN_STAGES
  static constexpr uint32_t V_OFF = K_OFF + ATTN_STAGES * TILE_BYTES;    // ATTN_STAGES
  static constexpr uint32_t BIAS_OFF = V_OFF + ATTN_STAGES * TILE_BYTES; // 2 x 128 fp32
  static constexpr uint32_t BAR_OFF = BIAS_OFF + 2u * 128u * 4u;
  static constexpr uint32_t NBARS = 21;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBARS * 8u;
  static constexpr uint32_t BYTES = MISC_OFF + 16u;
  static constexpr uint32_t ALLOC = BYTES + 1024u;  // slack for 1024-byte alignment
  static_assert(ALLOC <= 232448u, "exceeds the 227 KB shared-memory limit per block");
};

// barrier slots: ring stages indexed by t % 3, double buffers by t & 1
enum { B_QFULL = 0, B_KFULL0 = 1, B_VFULL0 = 4, B_EMPTY0 = 7, B_SFULL0 = 10, B_SFREE0 = 12,
       B_PFULL0 = 14, B_PVDONE0 = 16, B_BIAS0 = 18, B_DRAIN = 20 };

template <int D, bool DENSE, bool TRACE>
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
  const int tslot = !TRACE ? -1
                  : (blockIdx.x == 0 ? 0 : blockIdx.x == 1 ? 1 : blockIdx.x == gridDim.x / 3 ? 2 : -1);
  auto ev = [&](int e, int t) {
    if (TRACE && tslot >= 0 && t < TRACE_TILES)
      a.trace[((size_t)tslot * 16 + e) * TRACE_TILES + t] = clock64();
  };

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars[B_QFULL], 128);
    for (int b = 0; b < ATTN_STAGES; ++b) {
      mbar_init(&bars[B_KFULL0 + b], 128);  // 128 cp.async arrivals (K rows of a tile)
      mbar_init(&bars[B_VFULL0 + b], 128);  // 128 cp.async arrivals (V rows of a tile)
      mbar_init(&bars[B_EMPTY0 + b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_SFULL0 + b], 1);
      mbar_init(&bars[B_SFREE0 + b], 128);
      mbar_init(&bars[B_PFULL0 + b], 128);
      mbar_init(&bars[B_PVDONE0 + b], 1);
      mbar_init(&bars[B_BIAS0 + b], 128);  // each softmax thread writes its column's shift
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
  const uint32_t TM_P0 = tmem + 384;  // columns [384,448): 128 bf16 per row
  const uint32_t TM_P1 = tmem + 448;  // columns [448,512)

  if (warp >= 4 && warp < 8) {
    // ================================================================ producers
    const int p = tid - 128;       // 0..127
    const int u = p & 15;          // 16-byte unit within a 256-byte (D=128) row
    const int rsub = p >> 4;       // 0..7: this thread copies rows rsub, rsub+8, ...
    constexpr int UNITS = D / 8;   // 16-byte units per row
    const size_t plan_off = (size_t)blockIdx.x * a.s;
    const int nb = 128 >> a.bk_shift;  // sampled blocks per tile

    // Block indices of one tile, spread over the warp: lane e (+32k) holds the tile's
    // block e.  Loaded raw and coalesced one tile ahead (nothing branches on a loaded value
    // until the next tile, so the loads stay in flight), checked once per tile, and
    // broadcast to the copying lanes with shuffles; -1 marks padding or a rejected entry.
    constexpr int PAD = INT_MIN;
    int jc[4], jn[4];
    auto fetch = [&](int t, int (&jr)[4]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = lane + 32 * k;
        const int m = t * nb + e;
        jr[k] = (!DENSE && e < nb && m < a.s) ? __ldg(a.idx + plan_off + m) : PAD;
      }
    };
    auto check = [&](int (&jr)[4]) {
      bool bad = false;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool ok = jr[k] >= 0 && jr[k] < a.nK;
        bad |= (jr[k] != PAD) && !ok;
        jr[k] = ok ? jr[k] : -1;
      }
      if (bad) ab_flag(AB_ERR_DEVICE_CHECK);
    };
    if (!DENSE) {
      fetch(0, jc);
      check(jc);
    }

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

    int st = 0;  // t % ATTN_STAGES
    for (int t = 0; t < T; ++t) {
      if (!DENSE && t + 1 < T) fetch(t + 1, jn);  // in flight while this tile is issued
      if (t >= ATTN_STAGES &&
          !mbar_wait(&bars[B_EMPTY0 + st], (t / ATTN_STAGES - 1) & 1, abort_flag, a.timeout_ns))
        break;
      if (p == 0) ev(EV_COPY_START, t);
      const uint32_t kdst = sbase + L::K_OFF + st * L::TILE_BYTES;
      const uint32_t vdst = sbase + L::V_OFF + st * L::TILE_BYTES;
      int tokrow[16];  // token of each row this thread copies (-1: padding)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = rsub + 8 * i;  // row of the tile (= column of S)
        int tok;
        bool ok;
        if (DENSE) {
          tok = t * 128 + r;
          ok = tok < a.N;
        } else {
          const int ml = r >> a.bk_shift;  // block of the tile holding this row
          const int src = ml & 31;
          int j = __shfl_sync(0xffffffffu, jc[0], src);
          if (nb > 32) {  // warp-uniform: more than 32 blocks per tile (kv_block < 4)
            const int reg = ml >> 5;
#pragma unroll
            for (int k = 1; k < 4; ++k) {
              const int jk = __shfl_sync(0xffffffffu, jc[k], src);
              if (reg == k) j = jk;
            }
          }
          tok = j * a.bk + (r & (a.bk - 1));
          ok = j >= 0 && tok < a.N;
        }
        tokrow[i] = ok ? tok : -1;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // K rows, then V rows
        const uint16_t* gsrc = half ? a.V : a.K;
        const uint32_t dst = half ? vdst : kdst;
        if (u < UNITS) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = rsub + 8 * i;
            const int tok = tokrow[i];
            const size_t goff = head_off + (size_t)(tok >= 0 ? tok : 0) * D + u * 8;
            cp_async_16(dst + (u >> 3) * L::CHUNK_BYTES + sw128_off(r, u & 7), gsrc + goff,
                        tok >= 0 ? 16u : 0u);
          }
        }
        if (a.debug_skip_arrive && t == 0) continue;  // test knob: never signal tile 0
        mbar_arrive_cpasync(&bars[(half ? B_VFULL0 : B_KFULL0) + st]);
      }
      if (!DENSE && t + 1 < T) {
#pragma unroll
        for (int k = 0; k < 4; ++k) jc[k] = jn[k];
        check(jc);
      }
      st = (st + 1 == ATTN_STAGES) ? 0 : st + 1;
      if (p == 0) ev(EV_COPY_ISSUED, t);
    }
    cp_async_wait_all();
  } else if (warp == 8) {
    // ================================================================ MMA issuer
    // One thread issues QK(t) as soon as tile t has landed and S buffer t&1 is free, and
    // PV(t) as soon as P(t) is in tensor memory -- whichever is ready first (they touch
    // different tensor and shared memory), so PV never waits behind the next tile's copy.
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      // base descriptors; per 16-element K step only the start-address field moves
      // (stage b adds b * TILE_BYTES / 16 to the start-address field)
      const uint64_t dq = sdesc_sw128(sbase + L::Q_OFF, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + L::K_OFF, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sbase + L::V_OFF, L::CHUNK_BYTES, 1024);
      bool ok = mbar_wait(&bars[B_QFULL], 0, abort_flag, a.timeout_ns);
      int nqk = 0, npv = 0;              // next QK / PV to issue (npv < nqk)
      int sq = 0, sp = 0;                // their ring stages (t % 3)
      uint64_t t_last = globaltimer_ns();
      while (ok && npv < T) {
        bool progressed = false;
        if (npv < nqk && mbar_test(&bars[B_PFULL0 + (npv & 1)], (npv >> 1) & 1) &&
            mbar_test(&bars[B_VFULL0 + sp], (npv / ATTN_STAGES) & 1)) {
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t ap = (npv & 1) ? TM_P1 : TM_P0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 keys per MMA: 8 TMEM columns of P, 2 KB of V
            umma_f16_ts(TM_O, ap + kk * 8, dv0 + (uint64_t)((sp * L::TILE_BYTES + kk * 2048) >> 4), IDESC_PV,
                        (npv > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars[B_PVDONE0 + (npv & 1)]);
          umma_commit(&bars[B_EMPTY0 + sp]);
          ev(EV_PV, npv);
          ++npv;
          sp = (sp + 1 == ATTN_STAGES) ? 0 : sp + 1;
          progressed = true;
        }
        if (nqk < T && mbar_test(&bars[B_KFULL0 + sq], (nqk / ATTN_STAGES) & 1) &&
            (nqk < 2 || mbar_test(&bars[B_SFREE0 + (nqk & 1)], ((nqk >> 1) - 1) & 1))) {
          ev(EV_LANDED, nqk);
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t dS = (nqk & 1) ? TM_S1 : TM_S0;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t koff = (uint64_t)(((kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32) >> 4);
            umma_f16_ss(dS, dq + koff, dk0 + (uint64_t)(sq * L::TILE_BYTES >> 4) + koff, IDESC_QK,
                        kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[B_SFULL0 + (nqk & 1)]);
          ev(EV_QK, nqk);
          ++nqk;
          sq = (sq + 1 == ATTN_STAGES) ? 0 : sq + 1;
          progressed = true;
        }
        if (progressed) {
          t_last = globaltimer_ns();
        } else if (*abort_flag) {
          ok = false;
        } else if (globaltimer_ns() - t_last > a.timeout_ns) {
          ab_flag(AB_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        }
      }
      // drain: wait until every MMA issued above has completed before TMEM is freed
      umma_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0, abort_flag, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax (warps 0-3)
    const int r = tid;  // query row == TMEM lane; also the tile column whose shift it computes
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY;  // reference max (log2 domain)
    float l_run = 0.f;
    bool ok = true;
    const size_t plan_off = (size_t)blockIdx.x * a.s;
    const int nb = 128 >> a.bk_shift;
    // column r's plan entry for tile t as loaded (block index, log pi), -1 past the end of
    // the sample; both loads are unconditional so they stay in flight until the next tile
    auto entry = [&](int t, int& j, float& lp) {
      j = -1;
      lp = 0.f;
      if (!DENSE) {
        const int m = t * nb + (r >> a.bk_shift);
        if (m < a.s) {
          j = __ldg(a.idx + plan_off + m);
          lp = __ldg(a.logpi + plan_off + m);
        }
      }
    };
    int jcol, jnext = -1;
    float lcol, lnext = 0.f;
    entry(0, jcol, lcol);
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (r == 0) ev(EV_SM_START, t);
      {  // this thread's column of the shift row for tile t
        float b2;
        if (DENSE) {
          b2 = (t * 128 + r < a.N) ? 0.f : -INFINITY;
        } else {
          const bool valid = jcol >= 0 && jcol < a.nK && jcol * a.bk + (r & (a.bk - 1)) < a.N;
          b2 = valid ? -lcol * LOG2E : -INFINITY;
        }
        bias[st * 128 + r] = b2;
        mbar_arrive(&bars[B_BIAS0 + st]);
        if (t + 1 < T) entry(t + 1, jnext, lnext);
      }
      ok = mbar_wait(&bars[B_SFULL0 + st], (t >> 1) & 1, abort_flag, a.timeout_ns);
      if (r == 0) ev(EV_SM_SFULL, t);
      ok = ok && mbar_wait(&bars[B_BIAS0 + st], (t >> 1) & 1, abort_flag, a.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      if (r == 0) ev(EV_SM_READY, t);
      const float* bcol = bias + st * 128;
      const uint32_t sadr = (st ? TM_S1 : TM_S0) + lane_off;
      uint32_t zr[128];  // S, then the shifted logits, as raw bits
      tmem_ld_32x32b_x32(sadr + 0, *reinterpret_cast<uint32_t(*)[32]>(zr + 0));
      tmem_ld_32x32b_x32(sadr + 32, *reinterpret_cast<uint32_t(*)[32]>(zr + 32));
      tmem_ld_32x32b_x32(sadr + 64, *reinterpret_cast<uint32_t(*)[32]>(zr + 64));
      tmem_ld_32x32b_x32(sadr + 96, *reinterpret_cast<uint32_t(*)[32]>(zr + 96));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[B_SFREE0 + st]);
      if (r == 0) ev(EV_SM_LOADED, t);
      float* z = reinterpret_cast<float*>(zr);
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float4 b4 = *(const float4*)(bcol + c);
        z[c] = fmaf(z[c], a.scale_log2, b4.x);
        z[c + 1] = fmaf(z[c + 1], a.scale_log2, b4.y);
        z[c + 2] = fmaf(z[c + 2], a.scale_log2, b4.z);
        z[c + 3] = fmaf(z[c + 3], a.scale_log2, b4.w);
        mx[(c >> 2) & 7] = fmaxf(mx[(c >> 2) & 7], fmaxf(fmaxf(z[c], z[c + 1]), fmaxf(z[c + 2], z[c + 3])));
      }
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
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
      if (r == 0) ev(EV_SM_MAX, t);
      // P buffer st is free once PV(t-2) has completed
      if (t >= 2) {
        ok = mbar_wait(&bars[B_PVDONE0 + st], ((t >> 1) - 1) & 1, abort_flag, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      if (r == 0) ev(EV_SM_PBUF, t);
      const uint32_t padr = (st ? TM_P1 : TM_P0) + lane_off;
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) {  // 32 keys -> 16 TMEM columns of packed bf16 pairs
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = fast_exp2(z[32 * g + 2 * e] - mref);
          const float p1 = fast_exp2(z[32 * g + 2 * e + 1] - mref);
          ls[(2 * e) & 7] += p0;
          ls[(2 * e + 1) & 7] += p1;
          pk[e] = pack_bf16x2_rn(p0, p1);
        }
        tmem_st_32x32b_x16(padr + 16 * g, pk);
      }
      const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
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
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL0 + st]);
      if (lane == 0) ev(warp == 0 ? EV_SM_PDONE : EV_SM_PDONE_W1 + warp - 1, t);
      jcol = jnext;
      lcol = lnext;
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
  if (tid == 0) ev(EV_END, 0);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace abattn
