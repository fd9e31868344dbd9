/*
 * abattn.h -- C ABI of the B200 (sm_100a) AB-Attention hot path.
 *
 * AB-Attention (onedev.kr/papers/1521) makes video-DiT attention sparse in three
 * stages, each exported here as one asynchronous call:
 *
 *   ab_select(Q, K)            -> S          IBCS: block scores          (page section "how it differs")
 *   ab_plan(S, s, seed)        -> idx, logpi SIP: inclusion probabilities
 *                                            and systematic sampling     (page section "how to use")
 *   ab_attn(Q, K, V, idx, logpi) -> O        packed-tile attention with
 *                                            the -log(pi) logit shift    (page section "premises & limits")
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Layout.  Q, K, V, O are contiguous bf16 [B, H, N, d] (d fastest), raster
 *    token order.  nQ = ceil(N / q_block) query blocks, nK = ceil(N / kv_block)
 *    KV blocks.  The last query block and the last KV block may be partial.
 *  - Ownership.  The caller allocates and frees every buffer (device memory,
 *    e.g. from PyTorch).  The library never allocates, frees or synchronises,
 *    except ab_get_status, which synchronises the given stream.
 *  - Pointers.  All tensor pointers are device pointers, 16-byte aligned.
 *  - Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work and returns.
 *  - Errors.  The return value reports host-side validation and launch errors;
 *    nothing is enqueued when a call returns an error.  Problems detected on the
 *    device (a bounded wait that ran out, an out-of-range block index) set a
 *    device status word instead, read (and cleared) by ab_get_status.
 *  - Numerics.  bf16 inputs, fp32 accumulation.  Pooled keys and centroids are
 *    rounded once to bf16 (nearest-even) from exact fp64 means; S is fp32.
 */
#ifndef ABATTN_H
#define ABATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AB_OK = 0,
  AB_ERR_INVALID_ARG = -1,     /* null/misaligned pointer, bad size, s out of range   */
  AB_ERR_UNSUPPORTED = -2,     /* valid but not built: d not in {64,128}, q_block!=128 */
  AB_ERR_CUDA = -3,            /* a CUDA launch or runtime call failed                 */
  AB_ERR_DEVICE_TIMEOUT = -4,  /* a device-side bounded wait gave up                   */
  AB_ERR_WORKSPACE = -5,       /* workspace missing or smaller than ab_workspace_bytes */
  AB_ERR_NOT_IMPLEMENTED = -6, /* entry point present but not available in this build  */
  AB_ERR_DEVICE_CHECK = -7     /* a device-side range check failed (bad idx entry)     */
} ab_status;

/* Shape and method parameters, passed to every call.
 *   B, H, N, d    batch, heads, tokens, head dim (d in {64, 128})
 *   q_block       query block = MMA tile height; must be 128 ("128-token query blocks")
 *   kv_block      KV block: a power of two in [1, 128]; the page uses 4
 *   clusters      query clusters per query block, 1..8; the page uses 8
 *   kmeans_iters  Lloyd iterations after the segment-mean start, 0..4; the page uses 1
 *                 (0 = the position-based 16-query segment means of the ablation)
 *   head0, heads_total
 *                 head sharding (no counterpart on the page, which runs on one GPU):
 *                 this call covers heads [head0, head0 + H) of a layer of heads_total
 *                 heads.  heads_total = 0 means the call is the whole layer (head0 must
 *                 then be 0); otherwise 0 <= head0 and head0 + H <= heads_total.  Every
 *                 tensor argument holds only this call's heads ([B, H, ...]).  Each head
 *                 is computed independently, and the two places where the whole layer
 *                 matters use the whole layer's numbering: the planner's Philox row is
 *                 (b * heads_total + head0 + h) * nQ + i, and the selector cuts its
 *                 work (and so rounds S) as for B * heads_total heads.  So S, idx, logpi
 *                 and O of a slice are bitwise equal to the matching rows of one call
 *                 over the whole layer.  A zero-initialised struct is the whole layer.  */
typedef struct {
  int B, H, N, d;
  int q_block;
  int kv_block;
  int clusters;
  int kmeans_iters;
  int head0;
  int heads_total;
} ab_params;

/* Bytes of device workspace ab_select needs for `p` (pooled keys, centroids, shares and
 * per-centroid softmax statistics).  Writes *bytes; returns AB_ERR_INVALID_ARG /
 * AB_ERR_UNSUPPORTED for bad parameters.  Only the selector takes a workspace: the
 * planner and the attention kernel keep their working state on chip.                */
ab_status ab_workspace_bytes(const ab_params* p, size_t* bytes);

/* IBCS block scores ("how it differs" section of the AB-Attention page).
 * For every (b, h) and query block i: one k-means pass over the block's queries
 * (started from the contiguous segment means) gives `clusters` centroids c and
 * query shares w; every KV block j gets a pooled key kbar_j = mean of its keys; then
 *     S[b,h,i,j] = sum_c w_c * softmax_j( <c, kbar_j> / sqrt(d) )
 * with the softmax over all nK blocks of the head, so each row of S sums to 1.
 *   Q, K   bf16 [B,H,N,d] (device, read)
 *   S      fp32 [B,H,nQ,nK] (device, written)
 *   ws     device workspace of at least ab_workspace_bytes(p) bytes, 256-byte aligned;
 *          its contents are scratch and are overwritten.                              */
ab_status ab_select(const ab_params* p, const void* Q, const void* K, float* S,
                    void* ws, size_t ws_bytes, void* stream);

/* ab_select plus its intermediate results, for tests.  Each extra output may be NULL.
 *   labels int8  [B,H,nQ*128]       cluster of each query (-1 for rows beyond N)
 *   cent   bf16  [B,H,nQ,clusters,d] centroids (zero for empty clusters)
 *   w      fp32  [B,H,nQ,clusters]   query shares
 *   Kp     bf16  [B,H,nK,d]          pooled keys                                      */
ab_status ab_select_debug(const ab_params* p, const void* Q, const void* K, float* S,
                          void* ws, size_t ws_bytes, int8_t* labels, void* cent, float* w,
                          void* Kp, void* stream);

/* SIP plan ("how to use" section of the AB-Attention page).  Per row (b, h, i):
 * inclusion probabilities pi_j = min(1, lambda * S_j) with sum_j pi_j = s, computed in
 * 2^-32 fixed point (lambda = the smallest fp32 whose fixed-point sum reaches s; the
 * last non-saturated blocks are trimmed so the sum is exactly s), then systematic
 * sampling of exactly s distinct blocks with one Philox4x32-10 draw
 * (key = seed, counter = (row, offset_lo, offset_hi, 0), row = (b*H + h)*nQ + i for a
 * whole layer, (b*heads_total + head0 + h)*nQ + i for a head slice).
 * Blocks with pi = 1 are always sampled.  If fewer than s blocks have S > 0, all of
 * them and the lowest-index zero blocks are taken with pi = 1.
 *   S      fp32 [B,H,nQ,nK] (device, read); entries <= 0 or NaN count as 0
 *   s      1 <= s <= nK
 *   idx    int32 [B,H,nQ,s] (device, written): ascending block indices
 *   logpi  fp32  [B,H,nQ,s] (device, written): natural log of each block's pi (<= 0)  */
ab_status ab_plan(const ab_params* p, const float* S, int s, uint64_t seed, uint64_t offset,
                  int32_t* idx, float* logpi, void* stream);

/* Systematic sampling given target inclusion probabilities pi (fp32 [B,H,nQ,nK],
 * entries in [0, 1], rows summing to s).  pi is put through the same fixed-point step
 * as ab_plan (pi used as the score vector), so the draw has exactly s blocks and the
 * returned logpi are the probabilities actually used; when a row of pi sums to s the
 * rescale factor is 1 to within fp32 rounding.  Arguments as ab_plan.                */
ab_status ab_sample(const ab_params* p, const float* pi, int s, uint64_t seed,
                    uint64_t offset, int32_t* idx, float* logpi, void* stream);

/* ab_select followed by ab_plan (SIP), with the two stages overlapped across heads: the
 * B*H heads are cut into `groups` slices (0 = automatic: 1, i.e. no split, which measured
 * fastest on B200 at the Wan2.1-14B shape; at most 64 and at most B*H);
 * slice g is scored on `stream` and then planned on `stream2` while slice g+1 is scored,
 * so the planner's integer work overlaps the selector's tensor-core and exponential work.
 * Results are bit-identical to ab_select then ab_plan with the same arguments (the
 * planner's Philox counter uses each row's index in the whole tensor).  On return, work
 * enqueued later on `stream` runs after both stages; `stream2` must differ from `stream`
 * to overlap (NULL or equal: the two stages run one after the other on `stream`).  The
 * workspace is the one ab_select needs for the whole problem.  Arguments otherwise as
 * ab_select and ab_plan.                                                               */
ab_status ab_select_plan(const ab_params* p, const void* Q, const void* K, float* S, void* ws,
                         size_t ws_bytes, int s, uint64_t seed, uint64_t offset, int32_t* idx,
                         float* logpi, int groups, void* stream, void* stream2);

/* Planner variants for the ablations on the AB-Attention page (the selection rules SIP
 * is compared against).  Same arguments and output layout as ab_plan, plus `mode`:
 *   AB_PLAN_SIP         exactly ab_plan.
 *   AB_PLAN_SIP_NO_IPW  the same draw as ab_plan, but logpi = 0 for every block: the
 *                       sampled blocks enter attention without inverse-probability
 *                       reweighting.
 *   AB_PLAN_UNIFORM     ab_plan's fixed-point inclusion probabilities and systematic
 *                       draw on a constant score row (S is not read): pi_j = s / nK up
 *                       to the 2^-32 fixed point and the trimmed tail; logpi as ab_plan.
 *   AB_PLAN_TOPK        the s blocks with the largest S (deterministic; ties to the lower
 *                       block index; NaN ranks below every number, +0 above -0), logpi =
 *                       0; seed and offset are unused.
 * Returns AB_ERR_INVALID_ARG for an unknown mode.                                      */
typedef enum {
  AB_PLAN_SIP = 0,
  AB_PLAN_SIP_NO_IPW = 1,
  AB_PLAN_UNIFORM = 2,
  AB_PLAN_TOPK = 3
} ab_plan_mode;
ab_status ab_plan_variant(const ab_params* p, const float* S, int s, uint64_t seed,
                          uint64_t offset, int mode, int32_t* idx, float* logpi, void* stream);

/* Packed-tile sparse attention ("premises & limits" section of the AB-Attention page).
 * For each query q of query block i:
 *   O_q = sum_{j in idx, t in block j, t < N} e^{z_t} v_t / sum e^{z_t},
 *   z_t = q.k_t / sqrt(d) - logpi_j,
 * computed in one online-softmax pass over ceil(s*kv_block/128) tiles of 128 gathered
 * tokens (tcgen05 MMAs, fp32 accumulation in tensor memory, O rounded to bf16).
 *   idx, logpi  as produced by ab_plan: int32/fp32 [B,H,nQ,s]; each row's idx entries
 *               must lie in [0, nK) and be strictly ascending (so no block counts
 *               twice).  A validation pass before the attention records
 *               AB_ERR_DEVICE_CHECK in the status word for any row that breaks either
 *               rule.  Entries outside [0, nK) are never gathered (their block gets
 *               weight 0); beyond that, O of a flagged row is not specified.
 *   O           bf16 [B,H,N,d] (device, written)                                      */
ab_status ab_attn(const ab_params* p, const void* Q, const void* K, const void* V,
                  const int32_t* idx, const float* logpi, int s, void* O, void* stream);

/* Dense softmax attention through the same tile kernel (contiguous 128-token tiles, no
 * gather, no shift): the s = all-blocks reference path.                              */
ab_status ab_attn_dense(const ab_params* p, const void* Q, const void* K, const void* V,
                        void* O, void* stream);

/* Test and profiling hook (no counterpart on the page): ab_attn with
 *  - skip_first_arrival != 0: the producers of every CTA never signal their first tile;
 *    the waiting warps give up after timeout_ns, record AB_ERR_DEVICE_TIMEOUT in the
 *    status word, drain their copies, free tensor memory and exit (O is undefined);
 *  - timeout_ns: the limit of every bounded device wait (> 0);
 *  - trace (device, may be NULL; 8-byte aligned, 3*16*128 uint64, zeroed by the caller):
 *    a separately compiled traced kernel records clock64() for each pipeline event of
 *    tiles 0..127 of CTAs 0, 1 and gridDim/3, at trace[(slot*16 + event)*128 + tile];
 *    events (producer warps: 0, 1; MMA warp: 4, 5, 7, 12; softmax warps: the rest):
 *      0 the tile's copies start (its ring stage is free)   1 all its copies are issued
 *      2 S loaded from tensor memory                         3 exponentials done (P built)
 *      4 K rows and shifts landed (seen by the MMA warp)     5 QK MMAs issued
 *      6 the P buffer is free (PV two tiles back done)       7 PV MMAs issued
 *      8 softmax tile start                                  9 S ready (QK done)
 *      10 P stored by warp 0                                 11 CTA end (tile slot 0)
 *      12 V rows landed (seen by the MMA warp)               13, 14, 15 P stored by warps 1, 2, 3
 * With skip_first_arrival = 0 and trace = NULL it is ab_attn with another wait limit.   */
ab_status ab_attn_debug(const ab_params* p, const void* Q, const void* K, const void* V,
                        const int32_t* idx, const float* logpi, int s, void* O,
                        int skip_first_arrival, uint64_t timeout_ns, uint64_t* trace,
                        void* stream);

/* Synchronises `stream`, returns the device status word (AB_OK if no device-side problem
 * was recorded since the last call, else the first recorded code) and clears it.       */
ab_status ab_get_status(void* stream);

/* Static English description of a status code. */
const char* ab_status_string(ab_status s);

/* Library version, major*10000 + minor*100 + patch. */
int ab_version(void);

/* ab_select for callers that cannot provide a workspace.  The paper has no counterpart:
 * this is a packaging variant of ab_select, same inputs, same S.
 *
 * Who needs it: code that may not allocate device memory and has no scratch buffer to
 * pass -- e.g. a plugin whose host framework owns every device allocation and gives its
 * plugins no scratch allocator, or a serving loop whose memory plan is fixed at start-up
 * and must not call cudaMalloc/cudaFree (they synchronise the device) mid-flight.
 *
 * Instead of `ws`, the call uses one scratch array compiled into the library
 * (16 MiB per GPU, held from library load until process exit).  It allocates nothing
 * itself.  Shapes whose ab_workspace_bytes exceeds 16 MiB (about two Wan2.1 heads of
 * N = 75,600 at d = 128) are rejected with AB_ERR_WORKSPACE and a message on stderr;
 * use ab_select for them.
 *  - The first call on each device looks up the array's device address (with that device
 *    current) and caches it for the device's current CUDA context; make that first call
 *    before any stream capture.  A call in a new context of the device (after
 *    cudaDeviceReset, say) looks the address up again.
 *  - All calls on a device share the one array and it keeps the previous call's contents
 *    (every byte the selector reads is written earlier in the same call, so nothing has
 *    to be cleared).  Calls whose work overlaps on the GPU -- on different streams, or
 *    from different threads -- race on the array: serialise them.
 * Other arguments, errors and results are those of ab_select.                         */
ab_status ab_select_noalloc(const ab_params* p, const void* Q, const void* K, float* S,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ABATTN_H */
