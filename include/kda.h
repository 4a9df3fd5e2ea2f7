/*
 * kda.h -- C ABI of the B200 chunked Kimi Delta Attention (KDA) prefill library (libkda.so).
 *
 * The operation (FlashKDA README, CANNBot-DSL samples/flash_kda, sections 功能说明 and
 * 参数说明): for every sequence b and value head h, with q/k L2-normalised per row, beta =
 * sigmoid(beta_logit) and a per-channel log-decay g activated from the raw gate,
 *
 *     S_t = S_{t-1} Diag(exp(g_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   S_0 = initial_state
 *     o_t = scale * S_t q_t
 *
 * computed in 64-token chunks (gamma, K~ = gamma*K, K- = K/gamma, Q~ = scale*gamma*Q,
 * T = stril(diag(beta) K~ K-^T), (I+T)^-1, U, W, then a sequential pass of the state over the
 * chunks).  The gate activation, whose formula the pages do not print, is
 *
 *     g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :]))     (natural log).
 *
 * Calling pattern, mirroring flash_kda_metadata + flash_kda (FlashKDA README, 快速开始):
 *   1. kda_plan_size + kda_plan on the host: builds an int32 schedule from the shape, the
 *      layout and the valid lengths only (no tensor values).  Reusable for any call with the
 *      same shape and lengths (e.g. every layer of a model).
 *   2. copy the plan to the device; kda_workspace_size; allocate the workspace.
 *   3. kda_forward: asynchronous, enqueue-only on the given stream.
 *
 * Ownership: the caller owns every buffer.  The library never allocates, frees or synchronises
 * inside kda_forward.  All device pointers must be device memory of the current device.
 * Errors: every argument check happens on the host before anything is enqueued and is returned
 * synchronously; nothing is enqueued when a check fails.  Launch failures return KDA_ERR_CUDA.
 * Device-side problems (a plan that does not match the shape, a bounded wait that gave up) set
 * a status word in the workspace that kda_device_status reports.  No call traps or aborts.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
  KDA_OK = 0,
  KDA_ERR_NULL = 1,        /* a required pointer is NULL */
  KDA_ERR_LAYOUT = 2,      /* layout is not BNSD, BSND or TND */
  KDA_ERR_SHAPE = 3,       /* B < 1, S < 1, or a size does not fit the index types */
  KDA_ERR_HEADS = 4,       /* not 1 <= Nqk <= Nv with Nv % Nqk == 0 */
  KDA_ERR_DIM = 5,         /* D is neither 128 nor 64 */
  KDA_ERR_LOWER_BOUND = 6, /* lower_bound not in [-5, 0], or scale not finite */
  KDA_ERR_SEQLENS = 7,     /* cu_seqlens malformed (see kda_plan) */
  KDA_ERR_PLAN = 8,        /* plan buffer too small, corrupt, or built for another shape */
  KDA_ERR_ALIAS = 9,       /* initial_state aliases final_state, or out aliases an input */
  KDA_ERR_WORKSPACE = 10,  /* workspace NULL/too small/not 256-byte aligned */
  KDA_ERR_CUDA = 11,       /* a CUDA runtime call or a kernel launch failed */
  KDA_ERR_TIMEOUT = 12,    /* a bounded device-side wait gave up (reported by kda_device_status) */
  KDA_ERR_DEVICE = 13,     /* the current device is not an sm_100 GPU */
  KDA_ERR_ALIGN = 14,      /* q/k/v/g/out/state/workspace not 16-byte aligned (beta: 2-byte) */
  KDA_ERR_CAPACITY = 15    /* kda_forward_noalloc: problem needs more than its fixed scratch */
} kda_status_t;

/* Tensor layouts of q/k/v/g/beta/out (FlashKDA README, 参数说明):
 *   BNSD: q,k [B,Nqk,S,D]  v,g,out [B,Nv,S,D]  beta [B,Nv,S]
 *   BSND: q,k [B,S,Nqk,D]  v,g,out [B,S,Nv,D]  beta [B,S,Nv]
 *   TND : q,k [T,Nqk,D]    v,g,out [T,Nv,D]    beta [T,Nv]     (packed; S field = T)
 * All tensors are dense and contiguous in the order written. */
typedef enum { KDA_LAYOUT_BNSD = 0, KDA_LAYOUT_BSND = 1, KDA_LAYOUT_TND = 2 } kda_layout_t;

typedef struct {
  int32_t layout; /* kda_layout_t */
  int32_t B;      /* sequences: batch slots (BNSD/BSND) or len(cu_seqlens) - 1 (TND) */
  int32_t Nqk;    /* query/key heads */
  int32_t Nv;     /* value heads; value head h reads q/k head h / (Nv / Nqk) */
  int32_t S;      /* storage length per slot (BNSD/BSND) or total packed tokens T (TND) */
  int32_t D;      /* head dim, 128 or 64 (Dk = Dv = D); see kda_forward for D = 64 */
} kda_shape_t;

/* Chunk length of the method (tokens). */
#define KDA_CHUNK 64

/* Human-readable name of a status code (static storage, never NULL). */
KDA_API const char* kda_status_string(kda_status_t status);

/* Number of int32 words kda_plan writes for this shape (header + one record per
 * (sequence, value head) unit).  Validates the shape. */
KDA_API kda_status_t kda_plan_size(const kda_shape_t* shape, size_t* n_int32);

/* Build the schedule (the flash_kda_metadata equivalent, FlashKDA README 功能说明: built from
 * shapes, layout, valid lengths and the device's core count; reads no tensor values).
 *   cu_seqlens_host: host int32 [B+1], in every layout the prefix sums of the valid lengths:
 *     cu[0] == 0 and len_b = cu[b+1] - cu[b] >= 1, so the array is strictly increasing and
 *     cu[B] is the sum of the lengths.
 *     TND : required, and cu[B] == T (the packed row count).
 *     BNSD/BSND: optional (NULL = every length is S); each len_b is also <= S, so cu[B] <= B*S;
 *     sequence b then occupies storage rows [0, len_b) of slot b (FlashKDA README 约束说明).
 *     Anything else is KDA_ERR_SEQLENS.
 *   num_sms: multiprocessor count of the target device (>= 1); recorded in the plan.
 *   plan, n_int32: host output buffer and its capacity in int32 words.
 * Units are ordered longest first.  Pure host code; never touches the GPU.
 *
 * Schedule: when the units would leave more than half of num_sms idle, the plan may be
 * segmented (see kda_plan_segmented).  The segment length is the one a cost model, counted in
 * chunk-times on one SM, predicts fastest: waves of work items in the two passes, plus the
 * start-state chain.  Units run whole when that is predicted faster, and always when there
 * are more units. */
KDA_API kda_status_t kda_plan(const kda_shape_t* shape, const int32_t* cu_seqlens_host, int32_t num_sms,
                      int32_t* plan, size_t n_int32);

/* kda_plan with an explicit schedule: segment_chunks == 0 runs every unit whole;
 * segment_chunks > 0 cuts every unit into segments of that many 64-token chunks (the last one
 * shorter) that run in parallel, the chunk-parallel form of the state scan.  Per chunk the
 * state update is affine, S_next = S M + R with M = Diag(gamma_C) - W^T K^ and R = U^T K^
 * (the FlashKDA README's chunk equations, 功能说明, rearranged), so a segment maps its start
 * state S to S M_seg + R_seg.  kda_forward then runs three kernels: (1) every segment's
 * (M_seg, R_seg) as the final state from S = I with v = 0 and from S = 0 (the first segment of
 * a unit runs from its true initial state instead, writing its outputs); (2) the segment start
 * states, S_{s+1} = S_s M_s + R_s in fp32; (3) every later segment again from its start state,
 * writing outputs and, for a unit's last segment, final_state.  Results agree with the whole-unit
 * schedule within rounding.  segment_chunks < 0 is KDA_ERR_SHAPE. */
KDA_API kda_status_t kda_plan_segmented(const kda_shape_t* shape, const int32_t* cu_seqlens_host,
                                        int32_t num_sms, int32_t segment_chunks, int32_t* plan,
                                        size_t n_int32);

/* Device workspace bytes kda_forward needs for this plan (host plan): 256, plus 192 KiB per
 * segment after each unit's first under a segmented schedule. */
KDA_API kda_status_t kda_workspace_size(const int32_t* plan_host, size_t n_int32, size_t* bytes);

/* The forward pass (FlashKDA README, flash_kda): writes out and final_state.
 *   shape        : as given to kda_plan.
 *   plan_host    : the plan on the host (read for validation and launch sizing only).
 *   plan_dev     : the same n_int32 words in device memory (read by the kernels).
 *   q, k         : bf16 raw queries/keys (normalised in the op).
 *   v, g         : bf16 values and raw gate.
 *   beta         : bf16 raw write logits (sigmoid in the op).
 *   scale        : query scale, usually D^-0.5; must be finite.
 *   initial_state: fp32 [B,Nv,D(Dv),D(Dk)] or NULL for zeros; read-only.
 *   A_log        : fp32 [Nv];  dt_bias: fp32 [Nv,D];  lower_bound in [-5, 0].
 *   workspace    : device scratch of at least kda_workspace_size bytes, 256-byte aligned.
 *   out          : bf16, v's shape and layout.  Valid rows get the output (rounded to nearest
 *                  even); rows past a sequence's valid length are written as zeros.
 *   final_state  : fp32 [B,Nv,D,D]; must not overlap initial_state.
 * Rows of the inputs past a valid length are never read.  Asynchronous: returns once the
 * kernels are enqueued on `stream`.
 * Head dim: the FlashKDA README (约束说明) fixes D = 128; D = 64 is the small-head case that FLA
 * PR 656 ("[kda] add recursive block intra", its summary and timing table) benchmarks.  A D = 64
 * problem runs through the same kernels as D = 128 with the upper 64 channels of q, k, v and g
 * read as zeros (the tensor maps end at D), dt_bias and the states indexed with row length D,
 * and only the first D output channels stored: zero channels add nothing to the q/k norms,
 * the scores or the state, so the result is the D = 64 operator, at the cost of a D = 128 one. */
KDA_API kda_status_t kda_forward(const kda_shape_t* shape, const int32_t* plan_host,
                         const int32_t* plan_dev, size_t n_int32, const void* q, const void* k,
                         const void* v, const void* g, const void* beta, float scale,
                         const float* initial_state, const float* A_log, const float* dt_bias,
                         float lower_bound, void* workspace, size_t workspace_bytes, void* out,
                         float* final_state, kda_stream_t stream);

/* The affine summary of every unit (context parallelism, step 1).  Per chunk the state update
 * is affine in the start state (the FlashKDA README's chunk equations, 功能说明, rearranged):
 * S_next = S M_c + R_c with M_c = Diag(gamma_C) - W^T K^ and R_c = U^T K^.  Over all the tokens
 * a unit holds, S_end = S_start M + R; this call writes M (the final state from S = I with
 * v = 0) and R (the final state from S = 0) of every unit, without outputs.
 *   shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, A_log, dt_bias, lower_bound,
 *   workspace, workspace_bytes: as for kda_forward (scale is not needed: it weights only the
 *                  outputs).  Under a segmented plan every segment's pair of maps is computed in
 *                  parallel (segments after a unit's first into the workspace's state slots) and
 *                  a second kernel composes them in fp32, M = M_0 M_1 ..., R = (R_0 M_1 + R_1)
 *                  M_2 + ...; otherwise every unit runs whole, twice.
 *   M_out, R_out : fp32 [B,Nv,D(Dv),D(Dk)] each, caller-owned, 16-byte aligned; they must not
 *                  overlap each other or any input (KDA_ERR_ALIAS).
 * Errors as kda_forward.  Asynchronous on `stream`. */
KDA_API kda_status_t kda_forward_summary(const kda_shape_t* shape, const int32_t* plan_host,
                                         const int32_t* plan_dev, size_t n_int32, const void* q,
                                         const void* k, const void* v, const void* g,
                                         const void* beta, const float* A_log,
                                         const float* dt_bias, float lower_bound,
                                         void* workspace, size_t workspace_bytes, float* M_out,
                                         float* R_out, kda_stream_t stream);

/* Fold of affine state maps (context parallelism, step 2; the same step as the segmented
 * schedule's middle kernel): for every unit u,
 *     S = S_in[u];  for j = 0 .. n_steps-1:  S = S M[j][u] + R[j][u];  S_out[u] = S
 * in fp32.  Rank r of a context-parallel group starts its span from the fold over the maps of
 * ranks 0 .. r-1.
 *   units        : number of D x D states (>= 1), e.g. B * Nv.
 *   D            : 128 or 64.
 *   n_steps      : >= 0; 0 copies S_in (or zeros) to S_out.
 *   S_in         : fp32 [units][D][D] or NULL for zeros.
 *   M, R         : fp32; step j's maps are [units][D][D] at M + j*step_stride and
 *                  R + j*step_stride (may be NULL when n_steps == 0).
 *   step_stride  : floats between consecutive steps' maps; 0 means units*D*D (maps packed
 *                  step-major); else >= units*D*D and a multiple of 4 (KDA_ERR_SHAPE).  An
 *                  all-gather of [M; R] pairs is read in place with M, M + units*D*D and
 *                  step_stride = 2*units*D*D.
 *   S_out        : fp32 [units][D][D]; may be S_in itself, must not overlap it otherwise, nor M
 *                  or R (KDA_ERR_ALIAS).
 * All pointers are device memory, 16-byte aligned (KDA_ERR_ALIGN).  Errors: KDA_ERR_DIM,
 * _SHAPE, _NULL, _ALIGN, _ALIAS, _DEVICE, _CUDA.  Asynchronous on `stream`. */
KDA_API kda_status_t kda_state_chain(int32_t units, int32_t D, int32_t n_steps,
                                     const float* S_in, const float* M, const float* R,
                                     int64_t step_stride, float* S_out, kda_stream_t stream);

/* Synchronise `stream` and return the device-side status recorded in `workspace` by the last
 * kda_forward that used it (KDA_OK, KDA_ERR_PLAN or KDA_ERR_TIMEOUT), or KDA_ERR_CUDA. */
KDA_API kda_status_t kda_device_status(const void* workspace, kda_stream_t stream);

/* Bytes of the fixed, library-owned scratch that kda_forward_noalloc uses on each GPU. */
#define KDA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* kda_forward for callers that cannot allocate device memory.  The pages have no counterpart
 * of this call; it exists for callers that cannot provide a device workspace: a plugin
 * interface that hands over only the tensors, or a host runtime whose memory pool forbids
 * extra cudaMalloc calls (cudaMalloc can also synchronise the device).
 *
 * It runs exactly what kda_forward runs (the same kernels, schedule and results, D = 128 or
 * 64), with the same arguments minus workspace and workspace_bytes.  In place of the caller's
 * workspace the library uses one fixed scratch array of KDA_NOALLOC_SCRATCH_BYTES per GPU: a
 * static __device__ array that every GPU loading libkda.so holds until the process exits.  The
 * call allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - A plan whose kda_workspace_size exceeds KDA_NOALLOC_SCRATCH_BYTES is rejected with
 *     KDA_ERR_CAPACITY before anything is enqueued.  A whole-unit plan needs 256 bytes; a
 *     segmented plan adds 196,608 bytes per segment after each unit's first, so up to 341 such
 *     segments fit.
 *   - The first call on each device looks up the scratch's device address with that device
 *     current and caches it; make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array, which keeps the last call's contents
 *     (the call clears what must start at zero).  Calls whose kernels overlap on the GPU (two
 *     streams, or two host threads) race on it: serialise them.
 *   - The device status word lives at the start of the scratch: kda_noalloc_status reads it. */
KDA_API kda_status_t kda_forward_noalloc(const kda_shape_t* shape, const int32_t* plan_host,
                                         const int32_t* plan_dev, size_t n_int32, const void* q,
                                         const void* k, const void* v, const void* g,
                                         const void* beta, float scale,
                                         const float* initial_state, const float* A_log,
                                         const float* dt_bias, float lower_bound, void* out,
                                         float* final_state, kda_stream_t stream);

/* kda_device_status for kda_forward_noalloc: synchronise `stream` and return the device-side
 * status recorded in the current device's fixed scratch by the last kda_forward_noalloc there
 * (KDA_OK, KDA_ERR_PLAN or KDA_ERR_TIMEOUT), or KDA_ERR_CUDA.  Allocates nothing. */
KDA_API kda_status_t kda_noalloc_status(kda_stream_t stream);

/* The single-token decode step that follows a prefill: one step of the recurrence the chunked
 * forward computes in 64-token blocks (FlashKDA README, 功能说明; FLA PR 656, "[kda] add
 * recursive block intra", keeps the same recurrence as its naive token-by-token kernel):
 *     S <- S Diag(e^g);  S <- S + beta (v - S k^) k^T;  o = scale S q^
 * with kda_forward's in-op activations (q, k L2-normalised; beta = sigmoid(logit);
 * g = lower_bound * sigmoid(e^A_log[h] (g_raw + dt_bias[h,:]))), one token per sequence.
 *   B, Nqk, Nv, D: sequences, query/key heads, value heads (Nv % Nqk == 0; value head h reads
 *                  query/key head h / (Nv / Nqk)), head dim (128 or 64).
 *   q, k         : bf16 [B, Nqk, D];  v, g: bf16 [B, Nv, D];  beta: bf16 [B, Nv] (logits).
 *   scale        : finite;  A_log: fp32 [Nv];  dt_bias: fp32 [Nv, D];  lower_bound in [-5, 0].
 *   state_in     : fp32 [B, Nv, D(Dv), D(Dk)], or NULL for zeros.
 *   state_out    : fp32 [B, Nv, D, D]; may be state_in itself (the update is done in place, each
 *                  state row read before it is written) but must not overlap it otherwise.
 *   out          : bf16 [B, Nv, D], rounded to nearest even.
 * The caller owns every buffer; the call allocates nothing.  Pointers are device memory, 16-byte
 * aligned (beta 2-byte).  Errors: KDA_ERR_DIM, _SHAPE, _HEADS, _NULL, _LOWER_BOUND (also a
 * non-finite scale), _ALIGN, _ALIAS (an output overlapping an input or the other output),
 * _DEVICE (not sm_100), _CUDA (launch failure).  Asynchronous on `stream`. */
KDA_API kda_status_t kda_decode(int32_t B, int32_t Nqk, int32_t Nv, int32_t D, const void* q,
                                const void* k, const void* v, const void* g, const void* beta,
                                float scale, const float* state_in, const float* A_log,
                                const float* dt_bias, float lower_bound, void* out,
                                float* state_out, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
