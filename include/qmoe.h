/*
 * qmoe.h -- C ABI of libqmoe.so: forward pass of a quantised top-k routed
 * Mixture-of-Experts FFN layer on one NVIDIA B200 (sm_100a).
 *
 * What the layer computes (sources are the five web pages the method is
 * described on; each is cited by its title and section):
 *
 *   1. Router.  z[t,e] = sum_i x[t,i] * Wr[e,i] + b[e] in fp32; the k experts
 *      with the largest z are selected (descending z, lower index first on
 *      ties); the gates are the softmax over all E logits, renormalised over
 *      the k selected experts.
 *      ("Quantized Mixture of Experts (Q-MoE)", section 3 "Components",
 *      gating network with top-k routing; "FineRMoE", Sparse Sum Layer
 *      paragraph: softmax probabilities are the mixing weights.)
 *   2. Expert-centric schedule.  Every (token, slot) decision is one task;
 *      tasks are grouped by expert (ascending id) and sorted by token id
 *      inside each group.  counts[e], offsets[e] (exclusive prefix sum),
 *      sorted_token[p] (token of task p) and inv_pos[t,j] (position of task
 *      (t,j)) describe the permutation.
 *      ("OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale",
 *      section 2.2, Expert-Centric Scheduling: task collection, grouping and
 *      sorting, grouped GEMM.)
 *   3. Grouped gate/up GEMM per expert with in-kernel dequantisation and a
 *      SwiGLU epilogue: h = silu(W1 x) * (W3 x).
 *   4. Grouped down GEMM: y = W2 h.
 *      ("FineRMoE", architecture paragraph: an expert is Up, Gate and Down
 *      matrices with an activation; "Quantized Mixture of Experts (Q-MoE)",
 *      sections 2-4: each expert is quantised on its own, INT8 / FP8 /
 *      INT4 / mixed precision, and only the selected experts run.)
 *   5. Combine: out[t] = sum_j g[t,j] * y[t,j] + sum_s y_shared[s,t], fp32
 *      accumulation in slot order, rounded to bf16.  Shared experts are
 *      always active with weight 1.
 *      ("OmniMoE ...", section 2.1: the shared dense MLP every input
 *      activates.)
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent,
 *     on the device that was current at qmoe_create), row-major, densely
 *     packed, at least 16-byte aligned.  The one exception is
 *     qmoe_forward_host, which takes host pointers.
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it; no call synchronises it except
 *     qmoe_create, qmoe_destroy, qmoe_forward_host and qmoe_check_error.
 *   - Arguments are validated before anything is launched; on an invalid
 *     argument nothing is enqueued and QMOE_ERR_INVALID is returned.  A
 *     failed CUDA call returns QMOE_ERR_CUDA.  qmoe_last_error() gives a
 *     thread-local message for the last failure.
 *   - A handle may be used from one host thread at a time.  Calls on the
 *     same handle that overlap on the GPU (different streams without
 *     ordering) race on its workspace.
 */
#ifndef QMOE_H_
#define QMOE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QMOE_OK = 0,
  QMOE_ERR_INVALID = 1,      /* bad argument (NULL, out-of-range size, unknown format) */
  QMOE_ERR_UNSUPPORTED = 2,  /* valid but not supported here (e.g. no sm_100 device) */
  QMOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  QMOE_ERR_OOM = 4,          /* device allocation failed in qmoe_create */
  QMOE_ERR_TIMEOUT = 5,      /* a kernel's bounded wait ran out (see qmoe_check_error) */
  QMOE_ERR_BOUNDS = 6        /* QMOE_DEBUG build only: a device-side bounds check failed */
} qmoe_status;

/* Expert weight formats ("Quantized Mixture of Experts (Q-MoE)", section 3,
 * Expert Quantizer: INT8, FP8, mixed; section 4: INT4/INT8).  All symmetric,
 * no zero point.  N is the number of output rows, K the reduction length. */
typedef enum {
  QMOE_W_INT8_PC = 1,     /* codes int8 [N][K]; scale fp32 [N]; w = q * s[n]              */
  QMOE_W_INT4_G128 = 2,   /* codes u8 [N][K/2], low nibble = even k, two's complement;
                             scale bf16 [N][K/128]; w = q * s[n][k/128]                    */
  QMOE_W_FP8_E4M3_PC = 3  /* codes u8 e4m3 [N][K]; scale fp32 [N]; w = e4m3(q) * s[n].
                             The NaN codes 0x7F/0xFF are not supported (read as +-480).    */
} qmoe_wfmt;

/* Layer shape.  d: hidden size; E: routed experts (1..256); k: experts per
 * token (1..min(E,16)); I: expert intermediate size; n_shared: always-on
 * shared experts (0..8); max_tokens: largest T any later call may pass.
 * d and I must be multiples of 128. */
typedef struct {
  int32_t d, E, k, I, n_shared, max_tokens;
} qmoe_config;

/* One expert's weights in the canonical layout above.  w13/s13 hold the
 * gate and up projections stacked: rows 0..I-1 are the gate matrix W1 (the
 * silu operand), rows I..2I-1 the up matrix W3; K = d.  w2/s2 hold the down
 * matrix W2: N = d rows, K = I. */
typedef struct {
  int32_t fmt;            /* qmoe_wfmt */
  const void* w13;
  const void* s13;
  const void* w2;
  const void* s2;
} qmoe_expert;

typedef struct qmoe_handle qmoe_handle;

/* Create a layer.  router_w: fp32 [E][d]; router_bias: fp32 [E] or NULL
 * (added to the logits, so it affects both selection and gate values);
 * experts: host array of E + n_shared descriptors (routed experts first).
 * The weights are copied and re-laid-out into memory the handle owns, so
 * the caller may free its buffers once this returns; the workspace for
 * max_tokens is allocated here as well.  Synchronises the current device.
 * On success *out receives the handle; on failure *out is set to NULL.
 * Compute type: a layer whose experts are all FP8 e4m3 runs its GEMMs on
 * fp16 inputs (the codes, x and the intermediate H convert to fp16 with at
 * least bf16's precision), so its activations and H must stay inside the
 * fp16 range (|v| < 65504); every other layer runs on bf16 inputs.  Both
 * accumulate in fp32. */
qmoe_status qmoe_create(const qmoe_config* cfg, const float* router_w, const float* router_bias,
                        const qmoe_expert* experts, qmoe_handle** out);

/* Stages 1-2 only, with every intermediate written to caller buffers.
 * Exactly one of x (bf16 [T][d]) and logits (fp32 [T][E], used as given:
 * no bias is added) is non-NULL.  Outputs: topk_idx int32 [T][k] (slot j
 * = j-th largest logit), topk_gate fp32 [T][k], counts int32 [E], offsets
 * int32 [E+1], sorted_token int32 [T*k], inv_pos int32 [T][k].
 * 1 <= T <= max_tokens. */
qmoe_status qmoe_route(qmoe_handle* h, const uint16_t* x, const float* logits, int32_t T,
                       int32_t* topk_idx, float* topk_gate, int32_t* counts, int32_t* offsets,
                       int32_t* sorted_token, int32_t* inv_pos, void* stream);

/* The whole forward, stages 1-5: x bf16 [T][d] -> out bf16 [T][d].
 * 1 <= T <= max_tokens.  Intermediates live in the handle's workspace. */
qmoe_status qmoe_forward(qmoe_handle* h, const uint16_t* x, int32_t T, uint16_t* out, void* stream);

/* qmoe_forward for callers whose activations are in host memory: copies
 * x_host (bf16 [T][d]) to the device, runs the forward and copies the
 * result back to out_host, all on `stream`, then synchronises `stream`.
 * Page-locked host buffers make the copies asynchronous and faster. */
qmoe_status qmoe_forward_host(qmoe_handle* h, const uint16_t* x_host, int32_t T, uint16_t* out_host,
                              void* stream);

/* Synchronise `stream` and report whether any kernel of this handle hit its
 * bounded-wait limit since the last check (QMOE_ERR_TIMEOUT) or, in the
 * QMOE_DEBUG build, failed a device-side bounds check (QMOE_ERR_BOUNDS,
 * reported first), then clear the flags.  Returns QMOE_OK otherwise. */
qmoe_status qmoe_check_error(qmoe_handle* h, void* stream);

/* 1 in the QMOE_DEBUG build of the library, else 0.  That build (a
 * stand-in for a device memory checker) checks every index the kernels take
 * from data (expert ids, token rows, schedule positions, output rows) before
 * it is used: a failed check skips the access and raises QMOE_ERR_BOUNDS in
 * the handle's error word instead of faulting.  Results are otherwise the
 * same bits as the normal build's.  The method has no counterpart to this. */
int32_t qmoe_debug_build(void);

/* Bound, in SM clock cycles, of every barrier wait inside the grouped GEMM
 * kernels of this handle (0 restores the default of 2^31, about a second).
 * A kernel whose wait runs out stops cleanly: it lets the copies and MMAs it
 * issued finish, frees its tensor memory and raises the handle's error word,
 * which qmoe_check_error reports as QMOE_ERR_TIMEOUT; its output is then
 * undefined.  A limit far below a kernel's normal waits (a few thousand
 * cycles) makes that path run on purpose, which is how failure detection is
 * tested; the next forward at the default limit is unaffected.  Takes effect
 * for forwards enqueued after the call.  cycles < 0 -> QMOE_ERR_INVALID. */
qmoe_status qmoe_set_wait_limit(qmoe_handle* h, int64_t cycles);

/* Per-kernel timing.  With enable != 0, later qmoe_forward calls record a
 * CUDA event pair around each launch on the caller's stream.
 * qmoe_profile_read synchronises, adds the elapsed milliseconds of every
 * recorded launch to ms[stage] (stage ids below; n = array length),
 * writes the number of forwards counted to *calls and resets the record. */
enum { QMOE_STAGE_ROUTER = 0, QMOE_STAGE_SCHEDULE = 1, QMOE_STAGE_GATE_UP = 2,
       QMOE_STAGE_DOWN = 3, QMOE_STAGE_COMBINE = 4, QMOE_NUM_STAGES = 5 };
qmoe_status qmoe_profile(qmoe_handle* h, int32_t enable);
qmoe_status qmoe_profile_read(qmoe_handle* h, float* ms, int32_t n, int32_t* calls);

/* Launches one qmoe_forward enqueues for T tokens (kernels only). */
int32_t qmoe_launches_per_forward(const qmoe_handle* h, int32_t T);

/* Free everything the handle owns.  NULL-safe.  Synchronises the device. */
qmoe_status qmoe_destroy(qmoe_handle* h);

/* Thread-local text of the last failure in this thread ("" if none). */
const char* qmoe_last_error(void);

/* Stage 1 (router logits, softmax, top-k, renormalised gates: the gating
 * network with top-k routing of "Quantized Mixture of Experts (Q-MoE)",
 * section 3 "Components", with the softmax mixing weights of "FineRMoE",
 * Sparse Sum Layer) without a handle and without allocating anything.  The
 * method as published has no counterpart to calling it this way: it exists for callers that cannot allocate
 * device memory at the point where they route, for example a serving loop
 * whose memory is entirely held by another allocator (a caching or arena
 * allocator that owns all of HBM), or one that must not take the device-wide
 * synchronisation that cudaMalloc / cudaFree imply in the middle of a step.
 * It computes exactly what qmoe_route computes for topk_idx / topk_gate
 * from x, with the same kernel.
 *
 * x: bf16 [T][d] (device, 16-byte aligned); router_w: fp32 [E][d] (device,
 * 16-byte aligned); router_bias: fp32 [E] (device) or NULL.  Outputs
 * (device): topk_idx int32 [T][k], topk_gate fp32 [T][k].  Requires
 * d % 128 == 0, 1 <= E <= 256, 1 <= k <= min(E, 16), T >= 1 and
 * T * E <= QMOE_ROUTE_STATIC_MAX_LOGITS; larger sizes are rejected with
 * QMOE_ERR_INVALID and nothing is enqueued.
 *
 * Scratch: the router's partial logits live in one fixed library-global
 * device array of QMOE_ROUTE_STATIC_SCRATCH_BYTES bytes per device (no
 * cudaMalloc, cudaFree or allocating library call is made; every scratch
 * element read is first written by the same call, so nothing is cleared).
 * The array's address is looked up once per device on the first call
 * (cudaGetSymbolAddress, which may load the module), so make that first
 * call before any stream capture begins.  Because the scratch is shared,
 * calls whose work may overlap on the same GPU (different streams, or
 * different host threads) race and give wrong results: serialise them. */
#define QMOE_ROUTE_STATIC_MAX_LOGITS (1 << 20)
#define QMOE_ROUTE_STATIC_SCRATCH_BYTES (4 * (1 << 20))
qmoe_status qmoe_route_topk_noalloc(const uint16_t* x, const float* router_w, const float* router_bias,
                                    int32_t T, int32_t d, int32_t E, int32_t k, int32_t* topk_idx,
                                    float* topk_gate, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QMOE_H_ */
