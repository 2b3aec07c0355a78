/*
 * pi_ffn.h -- C ABI of the predictor-gated, neuron-level sparse FFN decode
 * library (libpi_ffn.so, CUDA, sm_100a).
 *
 * The operation (PowerInfer, "Fast Large Language Model Serving with a
 * Consumer-grade GPU"; Elamur Research summary page, Summary and Interesting
 * ideas I3/I4; reboot-conseil overview, "A Locality-Centric Design"): for one
 * FFN layer and each decode token b,
 *   1. a small per-layer predictor scores every neuron:  h = P1 u_b,
 *      s = P2 h + bias;  neuron i is predicted active iff s_i > 0;
 *   2. the active ids are compacted into an ascending index list;
 *   3. only those rows of the up (and, for SwiGLU, gate) projection are read:
 *      phi_i = ReLU(W1_i . u + b1_i)  or  SiLU(Wg_i . u) * (Wu_i . u);
 *   4. only the matching rows of the neuron-major down projection W2^T are
 *      accumulated:  y_b = sum_{i in S_b} phi_i W2T_i.
 * Neurons are stored hottest first (offline reordering by firing frequency,
 * Interesting ideas I1), so [0, hot_prefix) may be read as a dense block and
 * the cold tail by index.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, caller-owned and borrowed for
 *    the duration of the call (or of the stream work it enqueues).  The
 *    library never allocates device memory; the caller allocates the
 *    workspace (size from pi_workspace_size) and every input and output.
 *    The one exception to the workspace rule is pi_decode_ffn_static, which
 *    uses a fixed-size device array of the library instead.
 *  - Row-major layouts.  fp16 is IEEE binary16.  int4g32: each neuron row is
 *    d/2 bytes of packed nibbles (element 2k in the low nibble of byte k,
 *    2k+1 in the high nibble) with one fp16 scale per 32 consecutive elements
 *    in a separate [f x d/32] array; value = scale * (q - 8).
 *  - Work is enqueued on the given stream (a cudaStream_t; NULL = legacy
 *    default stream) and is asynchronous; nothing synchronises the host
 *    except pi_get_device_status.  No call allocates; the entry points that
 *    take a workspace may be captured into a CUDA graph.
 *  - Argument errors are detected on the host before anything is launched
 *    and returned synchronously; nothing is enqueued then.  Problems only the
 *    device can see (an out-of-range id in a caller's list, a bounded wait
 *    that gave up) are recorded in a status word inside the workspace and
 *    read back with pi_get_device_status; kernels never trap.
 *  - Alignment: every pointer 16-byte aligned; d % 8 == 0 for fp16 weights,
 *    d % 32 == 0 for int4g32, d % 4 == 0 for fp32, rank % 8 == 0 (fp16
 *    predictor) or % 4 (fp32); d <= 16384, 1 <= batch <= 32.  Some kernels
 *    need more (32-byte aligned matrices, d a multiple of 64 or 256); a call
 *    whose arguments do not meet them runs on a slower kernel that computes
 *    the same result, never fails for it (see pi_decode_ffn).
 */
#ifndef PI_FFN_H
#define PI_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pi_stream_t; /* same type as cudaStream_t */

typedef enum pi_status {
  PI_OK = 0,
  PI_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum */
  PI_ERR_UNSUPPORTED = 2,   /* shape/type combination the kernels do not cover */
  PI_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
  PI_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, memset) */
  PI_ERR_TIMEOUT = 5,       /* a bounded device wait gave up (device status) */
  PI_ERR_DEVICE_STATUS = 6, /* device-side argument error, e.g. id >= d_ffn */
  PI_ERR_WORKSPACE = 7      /* workspace missing or smaller than required */
} pi_status;

typedef enum pi_act { PI_ACT_RELU = 0, PI_ACT_SWIGLU = 1 } pi_act;

typedef enum pi_wtype { PI_W_F32 = 0, PI_W_F16 = 1, PI_W_INT4G32 = 2 } pi_wtype;

/* Flags of pi_sparse_ffn / pi_decode_ffn / pi_decode_ffn_stack. */
enum {
  PI_FFN_ACCUMULATE = 1u, /* y += result instead of y = result (pi_sparse_ffn, pi_decode_ffn) */
  PI_FFN_HOT_DENSE = 2u,  /* read the hot prefix [0, hot_prefix) as one dense block */
  PI_FFN_HOT_INDEX = 4u   /* read the hot prefix by index like the tail */
  /* neither HOT flag: dense when the expected union density of the prefix,
     1 - (1 - hot_p_mean)^B, is at least 0.75; otherwise by index */
};

/* One FFN layer and its predictor.  All pointers: device memory, borrowed;
 * they must stay valid while the handle is used. */
typedef struct pi_ffn_desc {
  int d_model;    /* d */
  int d_ffn;      /* f, number of neurons */
  int rank;       /* r, predictor rank */
  int act;        /* pi_act */
  int wtype;      /* pi_wtype of w_up / w_gate / w_down_t.  The FFN input u is
                     fp32 when wtype == PI_W_F32, fp16 otherwise. */
  int ptype;      /* PI_W_F32 or PI_W_F16: type of p1 and p2 */
  int hot_prefix; /* H: neurons [0, H) are the hot prefix (0 = none); rounded
                     down to a multiple of 32 */
  float hot_p_mean; /* mean firing probability of the hot prefix (offline
                       profile), used only by the automatic dense/index choice */
  const void *w_up;     /* ReLU: W1 [f x d]; SwiGLU: W_up [f x d] */
  const void *w_gate;   /* SwiGLU: W_gate [f x d]; NULL for ReLU */
  const void *w_down_t; /* W2^T [f x d], neuron-major (row i = column i of W2) */
  const uint16_t *s_up, *s_gate, *s_down_t; /* int4g32 scales, fp16 [f x d/32]; else NULL */
  const float *b_up;    /* ReLU bias b1 [f] fp32; NULL for SwiGLU */
  const void *p1;       /* [r x d] */
  const void *p2;       /* [f x r] */
  const float *p_bias;  /* [f] fp32 predictor bias */
} pi_ffn_desc;

typedef struct pi_ffn *pi_ffn_t; /* opaque host-side handle; holds no device memory */

/* Validate a layer description and create a host handle (copies *desc).
 * Returns PI_ERR_INVALID_ARG / PI_ERR_UNSUPPORTED / PI_ERR_MISALIGNED on a bad
 * description; *out is set only on PI_OK. */
pi_status pi_ffn_create(const pi_ffn_desc *desc, pi_ffn_t *out);

/* Release a handle (NULL is ignored). */
void pi_ffn_destroy(pi_ffn_t h);

/* Bytes of device workspace needed to run any entry point on these layers at
 * batch <= max_batch on the current CUDA device (the size depends on its SM
 * count).  n_layers handles of the same d may share one workspace. */
pi_status pi_workspace_size(const pi_ffn_t *layers, int n_layers, int max_batch, size_t *bytes);

/* Zero a workspace (cudaMemsetAsync on the stream).  Required once before
 * first use; kernels leave it reusable afterwards (their counters and
 * barrier words return to their initial state at the end of every call, and
 * a workspace may serve calls of any batch up to the size it was sized for). */
pi_status pi_workspace_init(void *ws, size_t ws_bytes, pi_stream_t stream);

/* Predictor only (steps 1-2: the per-layer predictor of the summary page's
 * Summary, second paragraph, sized per layer as in Interesting ideas I3).
 * u: [B x d] (fp16, or fp32 for PI_W_F32).
 * idx: [B x f] int32, row b receives the ascending ids of token b's predicted
 * set in its first count[b] entries (the rest is left unspecified);
 * count: [B] int32. */
pi_status pi_predict(pi_ffn_t h, const void *u, int B, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                     pi_stream_t stream);

/* Sparse FFN over caller-supplied sets (steps 3-4: kernels that read the
 * rows and columns of the active neurons themselves, summary page,
 * Interesting ideas I4).  idx/count as produced by
 * pi_predict (ids must lie in [0, f); a list is used as a set: order and
 * repeats do not matter; an out-of-range id is skipped and sets the device
 * status PI_ERR_DEVICE_STATUS).  y: [B x d] fp32 output.  flags: PI_FFN_*. */
pi_status pi_sparse_ffn(pi_ffn_t h, const void *u, int B, const int32_t *idx, const int32_t *count, float *y,
                        unsigned flags, void *ws, size_t ws_bytes, pi_stream_t stream);

/* Whole single-layer decode step (steps 1-4, the predictor-gated FFN of the
 * summary page's Summary, second paragraph) from the FFN input u.  y: [B x d]
 * fp32.  idx/count: optional outputs as in pi_predict (NULL to skip).
 * Execution (the same for the predictor and sparse-FFN entry points where it
 * applies):
 *  - batch 1, fp16/int4 weights (d <= 8192): one persistent fused kernel;
 *  - batch 2..8, fp16 weights and predictor (d % 64 == 0, rank a multiple
 *    of 64 up to 1024, weight and predictor matrices 32-byte aligned):
 *    tensor-core (mma.sync) predictor kernel and one persistent FFN kernel
 *    over the union of the tokens' sets;
 *  - batch 9..32 with fp16 weights, or 2..32 with int4 weights (fp16
 *    predictor; int4: d % 256 == 0): tcgen05 GEMMs over the 128-neuron tiles
 *    that hold a predicted neuron of some token; for int4 batches of 2..8
 *    that meet the predictor conditions above, the batch predictor kernel
 *    replaces the two predictor GEMMs;
 *  - otherwise: CUDA-core predictor, compaction, gather and reduction kernels.
 * Results agree within the stated tolerances whichever path runs. */
pi_status pi_decode_ffn(pi_ffn_t h, const void *u, int B, float *y, int32_t *idx, int32_t *count, unsigned flags,
                        void *ws, size_t ws_bytes, pi_stream_t stream);

/* Stacked decode through L layers of the same d_model (all fp16 or int4g32
 * weights).  The pages show no normalisation; the pre-FFN RMS norm below is
 * this library's reading (the residual stream of a plain stack grows
 * without bound): for each layer l, u = fp16(x / sqrt(mean(x^2) + 1e-6)) per token,
 * then steps 1-4, then the residual add x += y.  x: [B x d] fp32, in/out.
 * idx_trace: optional [L x B x f_max] int32 (layer l, token b at
 * (l*B + b)*f_max), count_trace: optional [L x B]. */
pi_status pi_decode_ffn_stack(const pi_ffn_t *layers, int L, float *x, int B, int32_t *idx_trace,
                              int32_t *count_trace, unsigned flags, void *ws, size_t ws_bytes, pi_stream_t stream);

/* Size in bytes of the library's file-scope device scratch array, the only
 * device memory pi_decode_ffn_static uses besides its arguments. */
#define PI_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* pi_decode_ffn at batch 1 without a caller workspace and without allocating.
 * The pages have no counterpart: this is an integration entry point only.
 *
 * Who needs it: callers that cannot call cudaMalloc (or own no device
 * allocator) at decode time -- a plugin inside a runtime that hands out no
 * device memory, an engine whose caching allocator has reserved all of HBM
 * for weights and KV cache, or a latency-critical loop where cudaMalloc may
 * synchronise the device.  Instead of a workspace, the call uses a
 * PI_STATIC_SCRATCH_BYTES file-scope __device__ array of this library.  It
 * calls no cudaMalloc / cudaFree or allocating library routine.
 *
 * u: [d] (fp16, or fp32 for PI_W_F32 layers); y: [d] fp32; idx/count:
 * optional [f] / [1] int32 outputs as in pi_predict; flags: PI_FFN_*.
 * dev_status: optional device int (4-byte aligned); when non-NULL it receives,
 * in stream order, this call's device-side status (PI_OK, PI_ERR_TIMEOUT, ...).
 * It is the only way to see a device-side error of this entry point: there is
 * no caller workspace to read with pi_get_device_status, and the next call
 * clears the scratch status word.
 *
 * Limits and behaviour:
 *  - The layer's batch-1 scratch (status words, h, mask words, union lists
 *    and, per SM, one fp32 and one tagged 8-byte partial row of d entries)
 *    must fit PI_STATIC_SCRATCH_BYTES; otherwise the call returns
 *    PI_ERR_WORKSPACE and launches nothing.  On a 148-SM B200 this admits
 *    d_model <= 9357 at d_ffn = 28672 and rank 1024, i.e. every OPT-7B- to
 *    LLaMA2-70B-shaped layer (d_model <= 8192).
 *  - The first call on each device (and again after a device reset) does
 *    the set-up: it looks up the array's device address with the device
 *    current.  Make that first call before any stream capture.  Each call
 *    clears the scratch status and barrier words on the stream before its
 *    kernels; the fused kernel's exchange words are never cleared (their
 *    tags advance with every launch).
 *  - There is one scratch array per device: calls that overlap on the GPU
 *    (other streams, other host threads) race on it and give wrong results.
 *    Serialise them, e.g. on one stream. */
pi_status pi_decode_ffn_static(pi_ffn_t h, const void *u, float *y, int32_t *idx, int32_t *count, unsigned flags,
                               int *dev_status, pi_stream_t stream);

/* Test support for the device-side failure reporting; not part of the decode
 * path (the pages have no counterpart).  It makes the following batch-1 fused
 * launches of this process exercise their bounded waits without any fault:
 * entry withhold_row of the predictor's h (0 <= withhold_row < rank) is never
 * published, so every CTA's wait for h runs out after limit_us microseconds;
 * each launch then records PI_ERR_TIMEOUT in the workspace status word and
 * completes (its outputs are unspecified).  withhold_row = -1 with
 * limit_us = 0 restores normal operation; limit_us alone (withhold_row = -1)
 * only shortens the limit.  Returns PI_ERR_INVALID_ARG for withhold_row < -1,
 * or for a withheld entry without a limit.  Not thread-safe; set it while no
 * call is running. */
pi_status pi_debug_wait_fault(int withhold_row, unsigned limit_us);

/* Synchronise the stream, read and clear the workspace status word.  *code is
 * PI_OK or the first device-side error recorded since the last read. */
pi_status pi_get_device_status(void *ws, pi_stream_t stream, int *code);

/* Static description of a status code (never NULL). */
const char *pi_status_string(pi_status s);

#ifdef __cplusplus
}
#endif

#endif /* PI_FFN_H */
