// C ABI of the AB-Attention hot path: argument validation, workspace carving and
// kernel launches.  All kernels live in the included headers (one translation unit,
// one device status word).
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include <cudaTypedefs.h>

#include "abattn.h"
#include "attn.cuh"
#include "common.cuh"
#include "plan.cuh"
#include "select.cuh"

using namespace abattn;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded device wait

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

int ilog2_exact(int v) {
  int s = 0;
  while ((1 << s) < v) ++s;
  return (1 << s) == v ? s : -1;
}

struct Dims {
  int B, H, N, d, bk, C, iters;
  int h0, Ht;  // this call's heads are [h0, h0 + H) of a layer of Ht heads
  long long BH, nQ, nK;
};

ab_status check_params(const ab_params* p, Dims* out) {
  if (!p) return AB_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1 || p->d < 1) return AB_ERR_INVALID_ARG;
  if (p->kv_block < 1 || p->kv_block > 128 || ilog2_exact(p->kv_block) < 0) return AB_ERR_INVALID_ARG;
  if (p->clusters < 1 || p->kmeans_iters < 0) return AB_ERR_INVALID_ARG;
  if (p->q_block != 128) return AB_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return AB_ERR_UNSUPPORTED;
  if (p->clusters > CMAX || p->kmeans_iters > 4) return AB_ERR_UNSUPPORTED;
  if (p->head0 < 0 || p->heads_total < 0) return AB_ERR_INVALID_ARG;
  if (p->heads_total == 0 ? p->head0 != 0 : (long long)p->head0 + p->H > p->heads_total)
    return AB_ERR_INVALID_ARG;
  Dims d;
  d.B = p->B; d.H = p->H; d.N = p->N; d.d = p->d; d.bk = p->kv_block;
  d.C = p->clusters; d.iters = p->kmeans_iters;
  d.h0 = p->head0;
  d.Ht = p->heads_total > 0 ? p->heads_total : p->H;
  d.BH = (long long)p->B * p->H;
  d.nQ = (p->N + 127) / 128;
  d.nK = (p->N + p->kv_block - 1) / p->kv_block;
  // grid and index limits: every (b,h,query block) is one CTA of a 1-D grid and
  // element offsets must fit the kernels' size_t arithmetic; nK*2^32 must fit uint64; the
  // whole layer's plan rows number the 32-bit Philox counter word
  if (d.BH * d.nQ > 0x7fffffffLL || (long long)d.B * d.Ht * d.nQ > 0x7fffffffLL ||
      d.nK > (1LL << 30))
    return AB_ERR_UNSUPPORTED;
  *out = d;
  return AB_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Workspace {
  uint16_t* Kp;
  uint16_t* cent;
  float* w;
  float* stats;
  size_t bytes;
};

Workspace carve(const Dims& d, void* base) {
  Workspace ws;
  uint8_t* b = (uint8_t*)base;
  size_t off = 0;
  ws.Kp = (uint16_t*)(b + off);
  off = align256(off + (size_t)d.BH * d.nK * d.d * 2);
  ws.cent = (uint16_t*)(b + off);
  off = align256(off + (size_t)d.BH * d.nQ * CMAX * d.d * 2);
  ws.w = (float*)(b + off);
  off = align256(off + (size_t)d.BH * d.nQ * CMAX * 4);
  ws.stats = (float*)(b + off);  // per centroid row of each 32-query-block group: key-chunk slots
  off = align256(off + (size_t)d.BH * ((d.nQ + SC_QB - 1) / SC_QB) * SC_ROWS * SC_MAX_CHUNKS * 2 * 4);
  ws.bytes = off;
  return ws;
}

// Streaming multiprocessors of the current device (looked up once per device).
int device_sms() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

ab_status launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "abattn: CUDA error: %s\n", cudaGetErrorString(e));
    return AB_ERR_CUDA;
  }
  return AB_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (the library
// does not link libcuda directly).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)f;
  }();
  return fn;
}

// Unique id of the calling thread's current CUDA context (ids are never reused within a
// process, unlike context handles), through the driver entry points the runtime exposes.
// Per-device host caches of device objects key on it, so that a cache filled in a context
// that was destroyed since (cudaDeviceReset) is refilled instead of used.
bool current_context_id(unsigned long long* id) {
  static const auto fns = [] {
    void* get = nullptr;
    void* getid = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &get, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      get = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &getid, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      getid = nullptr;
    return std::make_pair((PFN_cuCtxGetCurrent_v4000)get, (PFN_cuCtxGetId_v12000)getid);
  }();
  if (!fns.first || !fns.second) return false;
  CUcontext ctx = nullptr;
  if (fns.first(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return fns.second(ctx, id) == CUDA_SUCCESS;
}

// Tensor map of a bf16 array [z][y][x] (x contiguous, x = d elements) read in boxes of
// 64 x box_y x 1 with the 128-byte swizzle; out-of-range rows read as zeros.
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_y) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {x, y, z};
  const cuuint64_t strides[2] = {x * 2, x * y * 2};  // bytes, dimensions 1 and 2
  const cuuint32_t box[3] = {64, box_y, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The score passes' work split is chosen for the whole layer's B * Ht heads, also when this
// launch covers a slice of them.
template <int D>
ab_status run_select(const Dims& d, const void* Q, const void* K, float* S, const Workspace& ws,
                     int8_t* labels, cudaStream_t st) {
  SelectArgs a;
  a.Q = (const uint16_t*)Q;
  a.K = (const uint16_t*)K;
  a.Kp = ws.Kp;
  a.cent = ws.cent;
  a.w = ws.w;
  a.stats = ws.stats;
  a.S = S;
  a.labels = labels;
  a.BH = (int)d.BH;
  a.N = d.N;
  a.nQ = (int)d.nQ;
  a.nK = (int)d.nK;
  a.bk = d.bk;
  a.C = d.C;
  a.iters = d.iters;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  const int sms = device_sms();
  const size_t units = (size_t)d.BH * d.nK * (D / 8);
  const size_t pool_cap = (size_t)sms * 32;
  const int pool_blocks = (int)((units + 255) / 256 < pool_cap ? (units + 255) / 256 : pool_cap);
  pool_kernel<D><<<pool_blocks, 256, 0, st>>>(a);
  kmeans_kernel<D><<<(unsigned)(d.BH * d.nQ), KM_THREADS, 0, st>>>(a);
  const ScoreSplit sp = score_split(d.BH, d.nQ, d.nK, (long long)d.B * d.Ht, sms);
  using SL = ScoreSmem<D>;
  if (cudaFuncSetAttribute(score_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SL::ALLOC) != cudaSuccess ||
      cudaFuncSetAttribute(score_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SL::ALLOC) != cudaSuccess)
    return launch_status();
  CUtensorMap tm_kp, tm_cent;
  if (!make_tmap_3d(&tm_kp, ws.Kp, D, (uint64_t)d.nK, (uint64_t)d.BH, 128) ||
      !make_tmap_3d(&tm_cent, ws.cent, D, (uint64_t)d.nQ * CMAX, (uint64_t)d.BH, SC_ROWS)) {
    fprintf(stderr, "abattn: cannot encode the selector's tensor maps\n");
    return AB_ERR_CUDA;
  }
  score_kernel<D, 1><<<sp.P, SC_THREADS, SL::ALLOC, st>>>(a, sp, tm_kp, tm_cent, kDefaultTimeoutNs);
  score_kernel<D, 2><<<sp.P, SC_THREADS, SL::ALLOC, st>>>(a, sp, tm_kp, tm_cent, kDefaultTimeoutNs);
  return launch_status();
}

// bh0: flattened (b, h) index of this launch's first head within the call (a launch over a
// slice of the call's heads, as ab_select_plan makes)
ab_status run_plan(const Dims& d, const float* S, int s, uint64_t seed, uint64_t offset,
                   int mode, int32_t* idx, float* logpi, cudaStream_t st, long long bh0 = 0) {
  PlanArgs a;
  a.nQ = (int)d.nQ;
  a.H = d.H;
  a.Ht = d.Ht;
  a.h0 = d.h0;
  a.bh0 = bh0;
  a.S = S;
  a.idx = idx;
  a.logpi = logpi;
  a.nK = (int)d.nK;
  a.s = s;
  a.seed = seed;
  a.offset = offset;
  a.mode = mode;
  const unsigned rows = (unsigned)(d.BH * d.nQ);
  if (mode == AB_PLAN_TOPK) {
    if (d.nK <= PLAN_SMEM_MAX_FLOATS) {
      const size_t smem = (size_t)d.nK * 4;  // the row's keys
      if (cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PLAN_SMEM_MAX_FLOATS * 4) != cudaSuccess)
        return launch_status();
      topk_kernel<true><<<rows, PLAN_THREADS, smem, st>>>(a);
    } else {
      topk_kernel<false><<<rows, PLAN_THREADS, 0, st>>>(a);
    }
    return launch_status();
  }
  {
    const int nK4 = (int)((d.nK + 3) / 4);
    const size_t smem = (size_t)(nK4 < PLAN_STAGE_FLOAT4S ? nK4 : PLAN_STAGE_FLOAT4S) * 16;  // staged part
    // per-device attributes, cheap enough to set on every launch; the largest
    // shared-memory carveout fits three staged rows per SM
    const bool whole = nK4 <= PLAN_STAGE_FLOAT4S;
    auto kern = whole ? plan_kernel<1> : plan_kernel<2>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PLAN_STAGE_FLOAT4S * 16) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return launch_status();
    kern<<<rows, PLAN_THREADS, smem, st>>>(a);
  }
  return launch_status();
}

template <int D, bool DENSE>
ab_status run_attn(const Dims& d, const void* Q, const void* K, const void* V, const int32_t* idx,
                   const float* logpi, int s, void* O, int debug_skip, uint64_t timeout_ns,
                   uint64_t* trace, cudaStream_t st) {
  AttnArgs a;
  a.Q = (const uint16_t*)Q;
  a.K = (const uint16_t*)K;
  a.V = (const uint16_t*)V;
  a.idx = idx;
  a.logpi = logpi;
  a.O = (uint16_t*)O;
  a.N = d.N;
  a.nQ = (int)d.nQ;
  a.nK = (int)d.nK;
  a.s = s;
  a.bk = d.bk;
  a.bk_shift = ilog2_exact(d.bk);
  a.ntiles = DENSE ? (int)((d.N + 127) / 128) : (int)(((long long)s * d.bk + 127) / 128);
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  a.sqrt_d = (float)sqrt((double)D);
  a.timeout_ns = timeout_ns;
  a.debug_skip_arrive = debug_skip;
  a.trace = trace;
  using L = AttnSmem<D>;
  const unsigned grid = (unsigned)(d.BH * d.nQ);
  if (!DENSE) {  // plan rows strictly ascending in [0, nK)
    const long long rows = d.BH * d.nQ;
    const long long warps_needed = rows;
    const long long cap = (long long)device_sms() * 8 * (PLAN_CHECK_THREADS / 32);
    const long long w = warps_needed < cap ? warps_needed : cap;
    plan_check_kernel<<<(unsigned)((w + PLAN_CHECK_THREADS / 32 - 1) / (PLAN_CHECK_THREADS / 32)),
                        PLAN_CHECK_THREADS, 0, st>>>(idx, rows, s, (int)d.nK);
  }
  if (trace) {
    if (cudaFuncSetAttribute(attn_kernel<D, DENSE, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::ALLOC) != cudaSuccess)
      return launch_status();
    attn_kernel<D, DENSE, true><<<grid, ATTN_THREADS, L::ALLOC, st>>>(a);
  } else {
    if (cudaFuncSetAttribute(attn_kernel<D, DENSE, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::ALLOC) != cudaSuccess)
      return launch_status();
    attn_kernel<D, DENSE, false><<<grid, ATTN_THREADS, L::ALLOC, st>>>(a);
  }
  return launch_status();
}

ab_status attn_common(const ab_params* p, const void* Q, const void* K, const void* V,
                      const int32_t* idx, const float* logpi, int s, void* O, bool dense,
                      int debug_skip, uint64_t timeout_ns, uint64_t* trace, void* stream) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return AB_ERR_INVALID_ARG;
  if (!dense) {
    if (!idx || !logpi || ((uintptr_t)idx & 3) || ((uintptr_t)logpi & 3)) return AB_ERR_INVALID_ARG;
    if (s < 1 || s > d.nK) return AB_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (d.d == 128)
    return dense ? run_attn<128, true>(d, Q, K, V, idx, logpi, s, O, debug_skip, timeout_ns, trace, st)
                 : run_attn<128, false>(d, Q, K, V, idx, logpi, s, O, debug_skip, timeout_ns, trace, st);
  return dense ? run_attn<64, true>(d, Q, K, V, idx, logpi, s, O, debug_skip, timeout_ns, trace, st)
               : run_attn<64, false>(d, Q, K, V, idx, logpi, s, O, debug_skip, timeout_ns, trace, st);
}

ab_status select_common(const ab_params* p, const void* Q, const void* K, float* S, void* ws,
                        size_t ws_bytes, int8_t* labels, void* cent, float* w, void* Kp,
                        void* stream) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(S)) return AB_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255)) return AB_ERR_WORKSPACE;
  Workspace wsp = carve(d, ws);
  if (ws_bytes < wsp.bytes) return AB_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  r = (d.d == 128) ? run_select<128>(d, Q, K, S, wsp, labels, st)
                   : run_select<64>(d, Q, K, S, wsp, labels, st);
  if (r != AB_OK) return r;
  // optional debug copies out of the workspace
  if (cent) {
    // [BH, nQ, CMAX, d] -> [BH, nQ, C, d]
    const size_t row = (size_t)d.d * 2;
    if (cudaMemcpy2DAsync(cent, row * d.C, wsp.cent, row * CMAX, row * d.C, (size_t)(d.BH * d.nQ),
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return launch_status();
  }
  if (w) {
    if (cudaMemcpy2DAsync(w, 4 * (size_t)d.C, wsp.w, 4 * (size_t)CMAX, 4 * (size_t)d.C,
                          (size_t)(d.BH * d.nQ), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return launch_status();
  }
  if (Kp) {
    if (cudaMemcpyAsync(Kp, wsp.Kp, (size_t)d.BH * d.nK * d.d * 2, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return launch_status();
  }
  return AB_OK;
}

ab_status plan_common(const ab_params* p, const float* S, int s, uint64_t seed, uint64_t offset,
                      int mode, int32_t* idx, float* logpi, void* stream) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (mode < AB_PLAN_SIP || mode > AB_PLAN_TOPK) return AB_ERR_INVALID_ARG;
  if (mode != AB_PLAN_UNIFORM && (!S || ((uintptr_t)S & 3))) return AB_ERR_INVALID_ARG;
  if (!idx || !logpi || ((uintptr_t)idx & 3) || ((uintptr_t)logpi & 3)) return AB_ERR_INVALID_ARG;
  if (s < 1 || s > d.nK) return AB_ERR_INVALID_ARG;
  return run_plan(d, S, s, seed, offset, mode, idx, logpi, (cudaStream_t)stream);
}

// Select then plan for heads [bh0, bh0 + n) of the flattened (b, h) order: the slice is a
// problem with B*H = n on offset pointers (every kernel of both stages works per (b, h)).
ab_status select_plan_slice(const Dims& d, long long bh0, long long n, const void* Q,
                            const void* K, float* S, void* ws, int s, uint64_t seed,
                            uint64_t offset, int32_t* idx, float* logpi, cudaStream_t st_sel,
                            cudaStream_t st_plan, cudaEvent_t ev) {
  Dims g = d;
  g.BH = n;
  const size_t qk = (size_t)bh0 * d.N * d.d;  // elements
  const void* Qg = (const uint16_t*)Q + qk;
  const void* Kg = (const uint16_t*)K + qk;
  float* Sg = S + (size_t)bh0 * d.nQ * d.nK;
  Workspace wsp = carve(g, ws);
  ab_status r = (d.d == 128) ? run_select<128>(g, Qg, Kg, Sg, wsp, nullptr, st_sel)
                             : run_select<64>(g, Qg, Kg, Sg, wsp, nullptr, st_sel);
  if (r != AB_OK) return r;
  if (st_plan != st_sel) {
    if (cudaEventRecord(ev, st_sel) != cudaSuccess || cudaStreamWaitEvent(st_plan, ev, 0) != cudaSuccess)
      return launch_status();
  }
  const size_t rows = (size_t)bh0 * d.nQ;
  return run_plan(g, Sg, s, seed, offset, AB_PLAN_SIP, idx + rows * s, logpi + rows * s, st_plan, bh0);
}

}  // namespace

extern "C" {

ab_status ab_workspace_bytes(const ab_params* p, size_t* bytes) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (!bytes) return AB_ERR_INVALID_ARG;
  *bytes = carve(d, nullptr).bytes;
  return AB_OK;
}

ab_status ab_select(const ab_params* p, const void* Q, const void* K, float* S, void* ws,
                    size_t ws_bytes, void* stream) {
  return select_common(p, Q, K, S, ws, ws_bytes, nullptr, nullptr, nullptr, nullptr, stream);
}

ab_status ab_select_debug(const ab_params* p, const void* Q, const void* K, float* S, void* ws,
                          size_t ws_bytes, int8_t* labels, void* cent, float* w, void* Kp,
                          void* stream) {
  return select_common(p, Q, K, S, ws, ws_bytes, labels, cent, w, Kp, stream);
}

ab_status ab_plan(const ab_params* p, const float* S, int s, uint64_t seed, uint64_t offset,
                  int32_t* idx, float* logpi, void* stream) {
  return plan_common(p, S, s, seed, offset, AB_PLAN_SIP, idx, logpi, stream);
}

}  // extern "C"

namespace {

// ab_select_plan's events (one per head group plus one for the end): created once per
// device context and reused by every call.  The mutex serialises the calls' enqueue
// sequences, so one call's records and waits never interleave with another host thread's.
constexpr int kSpMaxGroups = 64;
std::mutex g_sp_mu;
struct SpEvents {
  unsigned long long ctx = 0;
  bool made = false;
  cudaEvent_t ev[kSpMaxGroups + 1];
};
SpEvents g_sp_events[64];

// Events of the current device's context; call with g_sp_mu held.
ab_status select_plan_events(cudaEvent_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch_status();
  if (dev < 0 || dev >= 64) return AB_ERR_UNSUPPORTED;
  SpEvents& e = g_sp_events[dev];
  unsigned long long ctx = 0;
  if (e.made && current_context_id(&ctx) && e.ctx == ctx) {
    *out = e.ev;
    return AB_OK;
  }
  // first call in this context (the events of a context destroyed since are dropped); creating
  // an event also creates the device's context if there is none yet
  e.made = false;
  for (int g = 0; g <= kSpMaxGroups; ++g)
    if (cudaEventCreateWithFlags(&e.ev[g], cudaEventDisableTiming) != cudaSuccess) {
      for (int k = 0; k < g; ++k) cudaEventDestroy(e.ev[k]);
      return launch_status();
    }
  if (!current_context_id(&ctx)) {
    for (int g = 0; g <= kSpMaxGroups; ++g) cudaEventDestroy(e.ev[g]);
    fprintf(stderr, "abattn: cannot identify the current CUDA context\n");
    return AB_ERR_CUDA;
  }
  e.made = true;
  e.ctx = ctx;
  *out = e.ev;
  return AB_OK;
}

}  // namespace

extern "C" {

ab_status ab_select_plan(const ab_params* p, const void* Q, const void* K, float* S, void* ws,
                         size_t ws_bytes, int s, uint64_t seed, uint64_t offset, int32_t* idx,
                         float* logpi, int groups, void* stream, void* stream2) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(S)) return AB_ERR_INVALID_ARG;
  if (!idx || !logpi || ((uintptr_t)idx & 3) || ((uintptr_t)logpi & 3)) return AB_ERR_INVALID_ARG;
  if (s < 1 || s > d.nK) return AB_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255)) return AB_ERR_WORKSPACE;
  if (ws_bytes < carve(d, ws).bytes) return AB_ERR_WORKSPACE;
  cudaStream_t sa = (cudaStream_t)stream, sb = (cudaStream_t)stream2;
  if (!sb || sb == sa) return select_plan_slice(d, 0, d.BH, Q, K, S, ws, s, seed, offset, idx, logpi, sa, sa, nullptr);
  // automatic: no split.  On B200 at the Wan2.1-14B shape every split measured slower than
  // the two stages back to back (2 groups: 7.06 vs 6.89 ms; 8: 9.1 ms): both stages are
  // compute-bound and their CTAs do not fit on one SM together (shared memory).
  long long G = groups > 0 ? groups : 1;
  if (G > d.BH) G = d.BH;
  if (G > kSpMaxGroups) G = kSpMaxGroups;
  // events: one per group (select of group g done -> plan of group g may start), one for the
  // end.  A wait refers to the record enqueued last before it, so reusing the events across
  // calls is safe while the enqueue sequences do not interleave (the mutex).
  std::lock_guard<std::mutex> lock(g_sp_mu);
  cudaEvent_t* evs = nullptr;
  r = select_plan_events(&evs);
  if (r != AB_OK) return r;
  for (long long g = 0; g < G && r == AB_OK; ++g) {
    const long long b0 = d.BH * g / G, b1 = d.BH * (g + 1) / G;
    r = select_plan_slice(d, b0, b1 - b0, Q, K, S, ws, s, seed, offset, idx, logpi, sa, sb, evs[g]);
  }
  // the caller's stream sees every plan as done
  if (r == AB_OK && (cudaEventRecord(evs[G], sb) != cudaSuccess || cudaStreamWaitEvent(sa, evs[G], 0) != cudaSuccess))
    r = launch_status();
  return r;
}

ab_status ab_plan_variant(const ab_params* p, const float* S, int s, uint64_t seed, uint64_t offset,
                          int mode, int32_t* idx, float* logpi, void* stream) {
  return plan_common(p, S, s, seed, offset, mode, idx, logpi, stream);
}

ab_status ab_sample(const ab_params* p, const float* pi, int s, uint64_t seed, uint64_t offset,
                    int32_t* idx, float* logpi, void* stream) {
  return plan_common(p, pi, s, seed, offset, AB_PLAN_SIP, idx, logpi, stream);
}

ab_status ab_attn(const ab_params* p, const void* Q, const void* K, const void* V,
                  const int32_t* idx, const float* logpi, int s, void* O, void* stream) {
  return attn_common(p, Q, K, V, idx, logpi, s, O, false, 0, kDefaultTimeoutNs, nullptr, stream);
}

ab_status ab_attn_debug(const ab_params* p, const void* Q, const void* K, const void* V,
                        const int32_t* idx, const float* logpi, int s, void* O,
                        int skip_first_arrival, uint64_t timeout_ns, uint64_t* trace,
                        void* stream) {
  if (timeout_ns == 0) return AB_ERR_INVALID_ARG;
  if (trace && ((uintptr_t)trace & 7)) return AB_ERR_INVALID_ARG;
  return attn_common(p, Q, K, V, idx, logpi, s, O, false, skip_first_arrival ? 1 : 0, timeout_ns,
                     trace, stream);
}

ab_status ab_attn_dense(const ab_params* p, const void* Q, const void* K, const void* V, void* O,
                        void* stream) {
  return attn_common(p, Q, K, V, nullptr, nullptr, 0, O, true, 0, kDefaultTimeoutNs, nullptr, stream);
}

ab_status ab_get_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return launch_status();
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ab_status, sizeof(int)) != cudaSuccess) return launch_status();
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_ab_status, &zero, sizeof(int)) != cudaSuccess) return launch_status();
  return (ab_status)v;
}

const char* ab_status_string(ab_status s) {
  switch (s) {
    case AB_OK: return "ok";
    case AB_ERR_INVALID_ARG: return "invalid argument";
    case AB_ERR_UNSUPPORTED: return "unsupported configuration";
    case AB_ERR_CUDA: return "CUDA error";
    case AB_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case AB_ERR_WORKSPACE: return "workspace missing or too small";
    case AB_ERR_NOT_IMPLEMENTED: return "not implemented";
    case AB_ERR_DEVICE_CHECK: return "device-side range check failed";
  }
  return "unknown status";
}

int ab_version(void) { return 100; }

}  // extern "C"

// ------------------------------------------------------------------------------------
// ab_select_noalloc: the selector with its scratch compiled into the library.
//
// Some callers cannot give this library a workspace: a plugin inside a host framework
// that owns all device memory and exposes no scratch allocator to its plugins, or a
// serving loop whose device-memory plan is frozen at start-up and which must not call
// cudaMalloc/cudaFree (they synchronise the device and stall every stream) while
// requests are in flight.  For those callers the selector's scratch -- pooled keys,
// centroids, shares and per-centroid softmax statistics -- lives in one fixed array
// below instead of a caller buffer.
// ------------------------------------------------------------------------------------

// Capacity of the built-in scratch.  Every GPU that loads the library holds this much
// device memory until the process exits.
#define AB_NOALLOC_SCRATCH_BYTES (16u << 20)

static __device__ __align__(256) uint8_t g_ab_noalloc_scratch[AB_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side symbol is
// only a stand-in, so the address is looked up once per device (with that device
// current) and cached together with the id of the context it belongs to; a call in a
// newer context of the device (after cudaDeviceReset, the old address is gone) looks it
// up again.
ab_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch_status();
  if (dev < 0 || dev >= kMaxDevices) return AB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (g_noalloc_addr[dev] == nullptr || !have_ctx || g_noalloc_ctx[dev] != ctx) {
    void* addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_ab_noalloc_scratch);
    if (e != cudaSuccess || addr == nullptr) {
      fprintf(stderr, "abattn: cannot resolve the built-in scratch on device %d: %s\n", dev,
              cudaGetErrorString(e));
      cudaGetLastError();
      g_noalloc_addr[dev] = nullptr;
      return AB_ERR_CUDA;
    }
    // the lookup made the context current if it was not; cache under its id
    const bool have_now = have_ctx || current_context_id(&ctx);
    g_noalloc_addr[dev] = have_now ? addr : nullptr;  // no id: look up again next call
    g_noalloc_ctx[dev] = ctx;
    *out = addr;
    return AB_OK;
  }
  *out = g_noalloc_addr[dev];
  return AB_OK;
}

}  // namespace

extern "C" ab_status ab_select_noalloc(const ab_params* p, const void* Q, const void* K, float* S,
                                       void* stream) {
  Dims d;
  ab_status r = check_params(p, &d);
  if (r != AB_OK) return r;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(S)) return AB_ERR_INVALID_ARG;
  const size_t need = carve(d, nullptr).bytes;
  if (need > AB_NOALLOC_SCRATCH_BYTES) {
    fprintf(stderr,
            "abattn: ab_select_noalloc needs %zu bytes of scratch for this shape but the built-in "
            "array holds %u; call ab_select with a workspace instead\n",
            need, (unsigned)AB_NOALLOC_SCRATCH_BYTES);
    return AB_ERR_WORKSPACE;
  }
  void* base = nullptr;
  r = noalloc_scratch(&base);
  if (r != AB_OK) return r;
  const Workspace ws = carve(d, base);
  cudaStream_t st = (cudaStream_t)stream;
  return (d.d == 128) ? run_select<128>(d, Q, K, S, ws, nullptr, st)
                      : run_select<64>(d, Q, K, S, ws, nullptr, st);
}
