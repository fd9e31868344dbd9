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
// tokens t*128 .. t*128+127 of that sequence.  Roles (384 threads):
//   warps 4-10 producers: each tile's K rows and then its V rows by 16-byte cp.async into
//              128B-swizzled tiles, three stages deep (a stage is freed when PV of its
//              tile completes); zero rows for padding.  With the K rows, thread p < 128
//              writes the shift of tile row p into the stage's shift tile (below).  K and
//              V land on separate barriers so QK can start before V has arrived.  The
//              copies are issued through the same per-warp memory-instruction queues as
//              the softmax's special-function work; seven producer warps (two on three of
//              the four SM sub-partitions) keep the gather ahead of the softmax.
//   warp 11    allocates 512 TMEM columns; lane 0 issues the MMAs, whichever is ready:
//              S  = Q K_t^T + 1 b_t^T  (M=128, N=128; A = Q, then a constant A of ones,
//                                       both from tensor memory; B = K_t, then the
//                                       shift tile b_t, from shared memory)
//              O += P_t V_t            (M=128, N=d, K=128; A = P from tensor memory, B = V
//                                       read MN-major from the same tile layout)
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Loads its Q row into
//              tensor memory once, then per tile reads S (already shifted), takes the
//              exponentials against a running reference max, writes P as bf16 into tensor
//              memory and finally writes O / l.  The tile's maximum is computed only on a
//              warp's first tile or when the tile's row sum passes 2^64; the reference is
//              then raised (when the tile exceeds it by more than 2^8, decided per warp),
//              P written again and O rescaled.
// The shift -log(pi_j) of a sampled block (in logit units: -log(pi_j) * sqrt(d)) enters
// through the tensor cores as one more K=16 step: A = [1 1 0 ... 0] for every query row,
// B row n = [hi_n lo_n 0 ... 0] with hi = bf16(shift), lo = bf16(shift - hi), so S gains
// hi + lo (the shift to about 2^-17 relative) and the softmax threads touch no shared
// memory per tile.  Padding and out-of-range rows get hi = -2^100: their weight is 0.
// Tensor memory: S [0,128), O [128,128+d), P0 [256,320), P1 [320,384), Q [384,384+d/2),
// ones [448,464).  All waits are bounded; a stuck pipeline records AB_ERR_DEVICE_TIMEOUT
// and every role drains and exits.
#pragma once

#include <climits>

#include "common.cuh"

namespace abattn {

constexpr int ATTN_THREADS = 384;
constexpr int ATTN_PRODUCERS = 224;  // warps 4-10
constexpr int ATTN_ROW_GROUPS = ATTN_PRODUCERS / 16;  // 14: thread p copies rows p/16 + 14 i
constexpr int ATTN_STAGES = 3;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;
constexpr float LSUM_LIMIT = 18446744073709551616.0f;  // 2^64: a tile's row sum above it takes the max path
constexpr uint32_t SHIFT_PAD_BITS = 0xF180u;  // bf16 -2^100
constexpr float PAD_LOGIT_LOG2 = -1e20f;      // a tile maximum below this is all padding

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
  float sqrt_d;          // shift in logit units = -log(pi) * sqrt(d)
  uint64_t timeout_ns;
  int debug_skip_arrive; // test knob: producers skip the first tile's copy arrivals
  uint64_t* trace;       // TRACE builds: clock64 per (traced CTA, event, tile)
};

// Event tracing (TRACE builds only): CTAs 0, 1 and the one at a third of the grid record
// clock64() per tile for the events below into trace[((slot * 16) + event) * 128 + t].
enum { EV_COPY_START = 0, EV_COPY_ISSUED, EV_SM_LOADED, EV_SM_MAX, EV_LANDED, EV_QK,
       EV_SM_PBUF, EV_PV, EV_SM_START, EV_SM_READY, EV_SM_PDONE, EV_END, EV_V_LANDED,
       EV_SM_PDONE_W1, EV_SM_PDONE_W2, EV_SM_PDONE_W3, EV_COUNT };
constexpr int TRACE_TILES = 128;

template <int D>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = 128u * D * 2u;  // 128 rows x D bf16
  static constexpr uint32_t CHUNK_BYTES = 128u * 128u;   // one 64-column chunk of 128 rows
  // Shift tiles first: 128 x 16 bf16, K-major without swizzle, core matrices of 8 rows x
  // 16 bytes: elements 0..7 of row n at byte 16 n, elements 8..15 of row n at 2048 + 16 n.
  static constexpr uint32_t SHIFT_BYTES = 4096u;
  static constexpr uint32_t SHIFT_KHALF = 2048u;         // lbo: elements 8..15
  static constexpr uint32_t SHIFT_OFF = 0;                                  // ATTN_STAGES
  static constexpr uint32_t K_OFF = SHIFT_OFF + ATTN_STAGES * SHIFT_BYTES;  // ATTN_STAGES
  static constexpr uint32_t V_OFF = K_OFF + ATTN_STAGES * TILE_BYTES;       // ATTN_STAGES
  static constexpr uint32_t BAR_OFF = V_OFF + ATTN_STAGES * TILE_BYTES;
  static constexpr uint32_t NBARS = 17;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBARS * 8u;
  static constexpr uint32_t BYTES = MISC_OFF + 16u;
  static constexpr uint32_t ALLOC = BYTES + 1024u;  // slack for 1024-byte alignment
  static_assert(K_OFF % 1024u == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(ALLOC <= 232448u, "exceeds the 227 KB shared-memory limit per block");
};

// barrier slots: ring stages indexed by t % 3, P buffers by t & 1
enum { B_QFULL = 0, B_KFULL0 = 1, B_VFULL0 = 4, B_EMPTY0 = 7, B_SFULL = 10, B_SFREE = 11,
       B_PFULL0 = 12, B_PVDONE0 = 14, B_DRAIN = 16 };

// Validation of a plan handed to ab_attn (a separate pass, so the gather warps, which set
// the attention's pace, carry no extra work): each row must be strictly ascending, which
// makes every block count once, with entries in [0, nK).  One warp per row (grid-stride);
// a violation records AB_ERR_DEVICE_CHECK.  The attention itself masks entries outside
// [0, nK) (they are never gathered); the output of a row that breaks the order is not
// specified further.
constexpr int PLAN_CHECK_THREADS = 256;

__global__ void __launch_bounds__(PLAN_CHECK_THREADS) plan_check_kernel(const int32_t* idx, long long rows,
                                                                         int s, int nK) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (PLAN_CHECK_THREADS / 32);
  for (long long row = (long long)blockIdx.x * (PLAN_CHECK_THREADS / 32) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int32_t* r = idx + row * s;
    int carry = -1;  // last entry checked before (below every valid entry)
    bool bad = false;
    if ((s & 3) == 0 && ((uintptr_t)idx & 15u) == 0) {
      // 16-byte rows: four entries per lane, 128 per warp and step
      for (int m0 = 0; m0 < s; m0 += 128) {
        const int m = m0 + 4 * lane;
        const int4 v = m < s ? __ldg(reinterpret_cast<const int4*>(r + m)) : make_int4(0, 0, 0, 0);
        const int up = __shfl_up_sync(0xffffffffu, v.w, 1);
        const int prev = lane == 0 ? carry : up;
        carry = __shfl_sync(0xffffffffu, v.w, 31);
        bad |= m < s && (v.x < 0 || v.w >= nK || v.x <= prev || v.y <= v.x || v.z <= v.y || v.w <= v.z);
      }
    } else {
      for (int m0 = 0; m0 < s; m0 += 32) {
        const int m = m0 + lane;
        const int v = m < s ? __ldg(r + m) : INT_MAX;
        const int up = __shfl_up_sync(0xffffffffu, v, 1);
        const int prev = lane == 0 ? carry : up;
        carry = __shfl_sync(0xffffffffu, v, 31);
        bad |= m < s && (v < 0 || v >= nK || v <= prev);
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) ab_flag(AB_ERR_DEVICE_CHECK);
  }
}

template <int D, bool DENSE, bool TRACE>
__global__ void __launch_bounds__(ATTN_THREADS, 1) attn_kernel(AttnArgs a) {
  using L = AttnSmem<D>;
  static_assert(B_DRAIN < (int)L::NBARS, "barrier slots");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
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
    mbar_init(&bars[B_QFULL], 128);  // every softmax thread, once its Q row is in TMEM
    for (int b = 0; b < ATTN_STAGES; ++b) {
      mbar_init(&bars[B_KFULL0 + b], 128 + ATTN_PRODUCERS);  // shift stores + cp.async arrivals
      mbar_init(&bars[B_VFULL0 + b], ATTN_PRODUCERS);        // cp.async arrivals (V rows)
      mbar_init(&bars[B_EMPTY0 + b], 1);
    }
    mbar_init(&bars[B_SFULL], 1);
    mbar_init(&bars[B_SFREE], 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_PFULL0 + b], 128);
      mbar_init(&bars[B_PVDONE0 + b], 1);
    }
    mbar_init(&bars[B_DRAIN], 1);
    fence_mbar_init();
  }
  // zero the shift tiles once: per tile only the first 4 bytes of each row change
  for (uint32_t o = tid * 16u; o < ATTN_STAGES * L::SHIFT_BYTES; o += ATTN_THREADS * 16u)
    *(uint4*)(smem + L::SHIFT_OFF + o) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 11) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t TM_S = tmem;           // columns [0,128): S of the current tile
  const uint32_t TM_O = tmem + 128;     // columns [128, 128+D)
  const uint32_t TM_P0 = tmem + 256;    // columns [256,320): 128 bf16 per row
  const uint32_t TM_P1 = tmem + 320;    // columns [320,384)
  const uint32_t TM_Q = tmem + 384;     // columns [384, 384+D/2): the Q row as bf16 pairs
  const uint32_t TM_ONES = tmem + 448;  // columns [448,464): A of the shift step

  if (warp >= 4 && warp < 11) {
    // ================================================================ producers
    const int p = tid - 128;       // 0..223
    const int u = p & 15;          // 16-byte unit within a 256-byte (D=128) row
    const int rsub = p >> 4;       // 0..13: this thread copies rows rsub, rsub+14, ...
    constexpr int NROWS = (128 + ATTN_ROW_GROUPS - 1) / ATTN_ROW_GROUPS;  // 10
    constexpr int UNITS = D / 8;   // 16-byte units per row
    const size_t plan_off = (size_t)blockIdx.x * a.s;
    const int nb = 128 >> a.bk_shift;  // sampled blocks per tile

    // Plan entries of one tile, spread over the warp: lane e (+32k) holds the tile's
    // block e (index and log pi).  Loaded raw and coalesced one tile ahead (nothing
    // branches on a loaded value until the next tile, so the loads stay in flight),
    // checked once per tile, and broadcast to the copying lanes with shuffles; -1 marks
    // padding or a rejected entry.
    constexpr int PAD = INT_MIN;
    int jc[4], jn[4];
    float lc[4], ln[4];
    auto fetch = [&](int t, int (&jr)[4], float (&lr)[4]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = lane + 32 * k;
        const int m = t * nb + e;
        const bool in = !DENSE && e < nb && m < a.s;
        jr[k] = in ? __ldg(a.idx + plan_off + m) : PAD;
        lr[k] = in ? __ldg(a.logpi + plan_off + m) : 0.f;
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
    // entry of the block holding tile row r, from the lanes holding the tile's entries
    auto shfl_entry = [&](int r, const auto (&vals)[4]) {
      const int ml = r >> a.bk_shift;
      const int src = ml & 31;
      auto v = __shfl_sync(0xffffffffu, vals[0], src);
      if (nb > 32) {  // warp-uniform: more than 32 blocks per tile (kv_block < 4)
        const int reg = ml >> 5;
#pragma unroll
        for (int k = 1; k < 4; ++k) {
          const auto vk = __shfl_sync(0xffffffffu, vals[k], src);
          if (reg == k) v = vk;
        }
      }
      return v;
    };
    if (!DENSE) {
      fetch(0, jc, lc);
      check(jc);
    }

    int st = 0;  // t % ATTN_STAGES
    for (int t = 0; t < T; ++t) {
      if (!DENSE && t + 1 < T) fetch(t + 1, jn, ln);  // in flight while this tile is issued
      if (t >= ATTN_STAGES &&
          !mbar_wait(&bars[B_EMPTY0 + st], (t / ATTN_STAGES - 1) & 1, abort_flag, a.timeout_ns))
        break;
      if (p == 0) ev(EV_COPY_START, t);
      const uint32_t kdst = sbase + L::K_OFF + st * L::TILE_BYTES;
      const uint32_t vdst = sbase + L::V_OFF + st * L::TILE_BYTES;
      int jsh = 0;  // entry of tile row p & 127 (shuffles involve the whole warp)
      float lsh = 0.f;
      if (!DENSE) {
        jsh = shfl_entry(p & 127, jc);
        lsh = shfl_entry(p & 127, lc);
      }
      if (p < 128) {  // shift of tile row p (row p of the shift step's B): bf16 hi, lo
        bool valid;
        float sh = 0.f;
        if (DENSE) {
          valid = t * 128 + p < a.N;
        } else {
          const int j = jsh;
          const float lp = lsh;
          valid = j >= 0 && j * a.bk + (p & (a.bk - 1)) < a.N;
          sh = -lp * a.sqrt_d;
        }
        uint32_t bits = SHIFT_PAD_BITS;
        if (valid) {
          const uint32_t hi = pack_bf16x2_rn(sh, 0.f) & 0xFFFFu;
          const float rest = sh - __uint_as_float(hi << 16);
          bits = hi | (pack_bf16x2_rn(rest, 0.f) << 16);
        }
        *(uint32_t*)(smem + L::SHIFT_OFF + st * L::SHIFT_BYTES + p * 16) = bits;
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_KFULL0 + st]);
      }
      int tokrow[NROWS];  // token of each row this thread copies (-1: padding)
#pragma unroll
      for (int i = 0; i < NROWS; ++i) {
        const int r = min(rsub + ATTN_ROW_GROUPS * i, 127);  // row of the tile (= column of S)
        int tok;
        bool ok;
        if (DENSE) {
          tok = t * 128 + r;
          ok = tok < a.N;
        } else {
          const int j = shfl_entry(r, jc);
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
          for (int i = 0; i < NROWS; ++i) {
            const int r = rsub + ATTN_ROW_GROUPS * i;
            if (r >= 128) break;
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
        for (int k = 0; k < 4; ++k) {
          jc[k] = jn[k];
          lc[k] = ln[k];
        }
        check(jc);
      }
      st = (st + 1 == ATTN_STAGES) ? 0 : st + 1;
      if (p == 0) ev(EV_COPY_ISSUED, t);
    }
    cp_async_wait_all();
  } else if (warp == 11) {
    // ================================================================ MMA issuer
    // One thread issues QK(t) as soon as tile t (K rows and shifts) has landed and the
    // softmax has read S(t-1), and PV(t) as soon as P(t) is in tensor memory -- whichever
    // is ready first, so PV never waits behind the next tile's copy.
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      // base descriptors; per 16-element K step only the start-address field moves
      // (stage b adds b * TILE_BYTES / 16 to the start-address field)
      const uint64_t dk0 = sdesc_sw128(sbase + L::K_OFF, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sbase + L::V_OFF, L::CHUNK_BYTES, 1024);
      const uint64_t db0 = sdesc_noswizzle(sbase + L::SHIFT_OFF, L::SHIFT_KHALF, 128);
      bool ok = mbar_wait(&bars[B_QFULL], 0, abort_flag, a.timeout_ns);
      tc_fence_after();
      int nqk = 0, npv = 0;              // next QK / PV to issue (npv < nqk)
      int sq = 0, sp = 0;                // their ring stages (t % 3)
      int nv = 0;                        // TRACE: next tile whose V arrival is to be seen
      uint64_t t_last = globaltimer_ns();
      while (ok && npv < T) {
        bool progressed = false;
        // TRACE: V(nv) is polled once its K has landed and before PV(nv) is issued, so the
        // stage's barrier cannot be a phase ahead (V(nv + 3) waits for PV(nv))
        if (TRACE && nv < nqk && nv >= npv && nv < T &&
            mbar_test(&bars[B_VFULL0 + nv % ATTN_STAGES], (nv / ATTN_STAGES) & 1)) {
          ev(EV_V_LANDED, nv);
          ++nv;
        }
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
          if (TRACE && nv == npv) {  // seen here first
            ev(EV_V_LANDED, nv);
            ++nv;
          }
          ++npv;
          sp = (sp + 1 == ATTN_STAGES) ? 0 : sp + 1;
          progressed = true;
        }
        if (nqk < T && mbar_test(&bars[B_KFULL0 + sq], (nqk / ATTN_STAGES) & 1) &&
            (nqk == 0 || mbar_test(&bars[B_SFREE], (nqk - 1) & 1))) {
          ev(EV_LANDED, nqk);
          fence_proxy_async_smem();
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t koff = (uint64_t)(((kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32) >> 4);
            umma_f16_ts(TM_S, TM_Q + kk * 8, dk0 + (uint64_t)(sq * L::TILE_BYTES >> 4) + koff,
                        IDESC_QK, kk > 0 ? 1u : 0u);
          }
          umma_f16_ts(TM_S, TM_ONES, db0 + (uint64_t)(sq * L::SHIFT_BYTES >> 4), IDESC_QK, 1u);
          umma_commit(&bars[B_SFULL]);
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
    const int r = tid;  // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c = a.scale_log2;
    float m_run = -INFINITY;  // reference max (log2 domain)
    float l_run = 0.f;
    bool ok = true;
    {  // Q row r (zeros past the sequence end) and the ones of the shift step -> TMEM
      const uint4* qrow = (const uint4*)(a.Q + head_off + (size_t)(row0 + min(r, nvalid - 1)) * D);
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {  // 32 columns = 64 elements = 8 x 16 bytes
        uint32_t v[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 q4 = r < nvalid ? __ldg(qrow + c0 / 4 + k) : make_uint4(0u, 0u, 0u, 0u);
          v[4 * k] = q4.x;
          v[4 * k + 1] = q4.y;
          v[4 * k + 2] = q4.z;
          v[4 * k + 3] = q4.w;
        }
        tmem_st_32x32b_x32(TM_Q + lane_off + c0, v);
      }
      uint32_t ones[16];
      ones[0] = 0x3F803F80u;  // bf16 (1, 1): picks up hi and lo of each shift row
#pragma unroll
      for (int k = 1; k < 16; ++k) ones[k] = 0u;
      tmem_st_32x32b_x16(TM_ONES + lane_off, ones);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_QFULL]);
    }
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (r == 0) ev(EV_SM_START, t);
      ok = mbar_wait(&bars[B_SFULL], t & 1, abort_flag, a.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      if (r == 0) ev(EV_SM_READY, t);
      uint32_t zr[128];  // S (shifted, logit units) as raw bits
      tmem_ld_32x32b_x32(TM_S + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(zr + 0));
      tmem_ld_32x32b_x32(TM_S + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(zr + 32));
      tmem_ld_32x32b_x32(TM_S + lane_off + 64, *reinterpret_cast<uint32_t(*)[32]>(zr + 64));
      tmem_ld_32x32b_x32(TM_S + lane_off + 96, *reinterpret_cast<uint32_t(*)[32]>(zr + 96));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[B_SFREE]);
      if (r == 0) ev(EV_SM_LOADED, t);
      const float* z = reinterpret_cast<const float*>(zr);
      // P buffer st is free once PV(t-2) has completed
      if (t >= 2) {
        ok = mbar_wait(&bars[B_PVDONE0 + st], ((t >> 1) - 1) & 1, abort_flag, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      if (r == 0) ev(EV_SM_PBUF, t);
      const uint32_t padr = (st ? TM_P1 : TM_P0) + lane_off;
      // P = exp2(z c + nm) as packed bf16 pairs into tensor memory; returns the row sum
      auto emit = [&](float nm) {
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int g = 0; g < 4; ++g) {  // 32 keys -> 16 TMEM columns of packed bf16 pairs
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * g + 2 * e;
            const float p0 = fast_exp2(fmaf(z[c0], c, nm));
            const float p1 = fast_exp2(fmaf(z[c0 + 1], c, nm));
            ls[(2 * e) & 3] += p0;
            ls[(2 * e + 1) & 3] += p1;
            pk[e] = pack_bf16x2_rn(p0, p1);
          }
          tmem_st_32x32b_x16(padr + 16 * g, pk);
        }
        return (ls[0] + ls[1]) + (ls[2] + ls[3]);
      };
      // The exponentials are taken against the running reference m_run first; the tile's
      // maximum is needed only on a warp's first tile, or when a value came out more than
      // 2^57 above the reference (the row sum passes 2^64, or overflowed).  Values up to
      // 2^64 keep every sum far inside fp32 range, and softmax weights do not depend on the
      // reference, so the output is the same softmax.  Decided per warp: tcgen05.ld/st are
      // warp-collective, so when any row of the warp has to raise its reference, every row
      // of the warp moves to max(m_run, tile max) (alpha = 1 where nothing changes), its P
      // row is written again and the warp rescales O.
      float alpha = 1.f;
      bool rescale = false;
      float lsum = 0.f;
      bool redo = __any_sync(0xffffffffu, m_run == -INFINITY);
      if (!redo) {
        lsum = emit(-m_run);
        redo = __any_sync(0xffffffffu, !(lsum <= LSUM_LIMIT));
      }
      if (redo) {
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = z[k];
#pragma unroll
        for (int k = 8; k < 128; ++k) mx[k & 7] = fmaxf(mx[k & 7], z[k]);
        float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * c;
        if (mt < PAD_LOGIT_LOG2) mt = -INFINITY;  // every column of the tile is padding
        const bool need = mt > m_run + LAZY_RESCALE_LOG2;  // always true on a row's first finite tile
        rescale = __any_sync(0xffffffffu, need);
        if (rescale) {
          const float m_new = fmaxf(mt, m_run);
          if (m_new != -INFINITY) {
            alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
            m_run = m_new;
          }
        }
        lsum = emit((m_run == -INFINITY) ? 0.f : -m_run);
      }
      if (r == 0) ev(EV_SM_MAX, t);
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
          for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
          tmem_st_32x32b_x32(TM_O + lane_off + c0, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL0 + st]);
      if (lane == 0) ev(warp == 0 ? EV_SM_PDONE : EV_SM_PDONE_W1 + warp - 1, t);
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
          for (int k = 0; k < 32; k += 8) {
            uint4 o;
            o.x = pack_bf16x2_rn(__uint_as_float(v[k]) * inv, __uint_as_float(v[k + 1]) * inv);
            o.y = pack_bf16x2_rn(__uint_as_float(v[k + 2]) * inv, __uint_as_float(v[k + 3]) * inv);
            o.z = pack_bf16x2_rn(__uint_as_float(v[k + 4]) * inv, __uint_as_float(v[k + 5]) * inv);
            o.w = pack_bf16x2_rn(__uint_as_float(v[k + 6]) * inv, __uint_as_float(v[k + 7]) * inv);
            *(uint4*)(orow + c0 + k) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0) ev(EV_END, 0);
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace abattn
