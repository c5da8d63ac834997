/*
 * prox.h -- C ABI of the B200 (sm_100a) Prox two-stage sparse SwiGLU FFN.
 *
 * The method ("Prox: Training-Free FFN Activation Sparsity via Approximate
 * Intermediate-Channel Salience in LLMs"; sections cited below are those of
 * the Prox deep-dive blog post and of the translated arXiv HTML):
 *
 *   Stage 1 (blog, "Stage 1"): m_x = 1[|x| >= tau_x]; proxy branches
 *     u~ = Pi_in(x, W~_up, m_x), h~ = SiLU(Pi_in(x, W~_gate, m_x)) with
 *     symmetric per-row INT4 copies W~; s~ = u~ (.) h~; shared channel mask
 *     m_s = 1[|s~| >= tau_s].
 *   Stage 2 (blog, "Stage 2"): for the kept channels only, with the original
 *     bf16 weights and the full x: u = Pi_out(x, W_up, m_s),
 *     h = SiLU(Pi_out(x, W_gate, m_s)), s = u (.) h, y = Pi_in(s, W_down, m_s).
 *   Pi_in / Pi_out are the input- and output-sparse projections of the arXiv
 *   page, section 2.2; the SwiGLU FFN itself is its section 2.1.
 *
 * Conventions
 *   - Every pointer named "device" is CUDA device memory owned by the caller;
 *     the library never allocates, frees or keeps it. "host" pointers are
 *     ordinary host memory.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every
 *     call except prox_calibrate and prox_last_device_status is asynchronous
 *     on that stream and returns as soon as its kernels are enqueued.
 *   - Every device pointer (inputs, outputs, workspace) must be 16-byte
 *     aligned; optional outputs may be NULL.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched. No C++ exception crosses this interface.
 *   - Shapes: d_model and d_ff are multiples of 256 with 256 <= d_model <= 8192
 *     and 256 <= d_ff <= 262144; batch >= 0. Anything else is PROX_EINVAL.
 *   - The library runs on compute capability 10.0 devices (B200, sm_100a);
 *     any other current device gives PROX_EDEVICE.
 */
#ifndef PROX_H
#define PROX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum prox_status {
    PROX_OK = 0,
    PROX_EINVAL = 1,   /* bad argument (null pointer, shape, threshold, ...)  */
    PROX_ENOMEM = 2,   /* caller's workspace smaller than required           */
    PROX_ECUDA = 3,    /* a CUDA runtime call or launch failed               */
    PROX_ETIMEOUT = 4, /* a bounded device-side wait gave up (status word)   */
    PROX_EDEVICE = 5   /* current device is not compute capability 10.x      */
} prox_status;

/*
 * One FFN layer, all device pointers, caller-owned.
 *   w_up_cm, w_gate_cm : bf16 [d_ff][d_model]; row j is output channel j
 *                        (the pages' W_up[:, j]; nn.Linear weight layout).
 *   w_down             : bf16 [d_ff][d_model]; row j is W_down[j, :] (the
 *                        pages' orientation d_ff x d_model).
 *   q_up, q_gate       : INT4 proxies, uint8 [d_ff/256][d_model][128] (block-
 *                        tiled) as written by prox_quantize_proxy.
 *   s_up, s_gate       : fp32 [d_model] per-row proxy scales.
 * Every pointer must be 16-byte aligned.
 */
typedef struct prox_layer {
    int d_model;
    int d_ff;
    const uint16_t *w_up_cm;
    const uint16_t *w_gate_cm;
    const uint16_t *w_down;
    const uint8_t *q_up;
    const uint8_t *q_gate;
    const float *s_up;
    const float *s_gate;
    /* gate activation: PROX_ACT_SWIGLU (SiLU, the pages' SwiGLU FFN) or
       PROX_ACT_GEGLU (GELU(z) = z Phi(z), exact erf form: the GeGLU-style
       models of the blog's "Evidence" section); anything else is PROX_EINVAL */
    int activation;
    /* proxy kind: PROX_PROXY_INT4 (the method: q_up/q_gate INT4 tiles from
       prox_quantize_proxy, s_up/s_gate their scales) or PROX_PROXY_BF16 (the
       FP16/bf16-proxy ablation of the blog's "Evidence" section: q_up/q_gate
       are bf16 tiles [d_ff/256][d_model][256] from prox_bf16_proxy, the
       original weights; s_up/s_gate are unused and may be NULL) */
    int proxy_kind;
} prox_layer;

#define PROX_PROXY_INT4 0
#define PROX_PROXY_BF16 1

#define PROX_ACT_SWIGLU 0
#define PROX_ACT_GEGLU 1

/*
 * prox_quantize_proxy -- symmetric per-row INT4 proxy copy of one projection
 * (blog, "Stage 1": W~_up and W~_gate are symmetric per-row INT4 copies).
 *
 * Reading of "per-row": a row i of W in the pages' orientation
 * W in R^{d_model x d_ff}, i.e. one scale per input coordinate, so that the
 * input-sparse proxy product skips whole rows.
 *   scale_i = max_j |W[i,j]| / 7                        (fp32, round to nearest)
 *   q_ij    = clamp(round_half_even(W[i,j] / scale_i), -7, 7)  (fp32 division)
 *   an all-zero row gives scale 0 and q 0.
 * Output layout (block-tiled, the order the input-sparse proxy product
 * streams): q_out is uint8 [d_ff/256][d_model][128]; the 128-byte granule
 * q_out[c][i] holds the codes of row i for channels 256c .. 256c+255, byte m
 * holding channel 256c+2m in its low nibble and 256c+2m+1 in its high
 * nibble, each nibble holding q + 8 (offset binary, 1..15; 8 for q = 0).
 * A rejected input coordinate i thus skips one
 * contiguous granule per block. scale_out is fp32 [d_model].
 *   w_cm : device, bf16 [d_ff][d_model] (channel-major, as in prox_layer).
 * Errors: PROX_EINVAL on a null pointer or bad shape.
 */
prox_status prox_quantize_proxy(int d_model, int d_ff, const uint16_t *w_cm,
                                uint8_t *q_out, float *scale_out, void *stream);

/*
 * prox_bf16_proxy -- the bf16-proxy ablation's proxy: the weight itself,
 * block-tiled like the INT4 proxy so that a rejected input coordinate skips
 * one contiguous 512-byte granule per 256-channel block:
 *   q16_out[c][i][k] = w_cm[256c + k][i]   (uint16 bf16, [d_ff/256][d_model][256]).
 *   w_cm : device, bf16 [d_ff][d_model] (channel-major).
 * Errors: PROX_EINVAL on a null or misaligned pointer or a bad shape.
 */
prox_status prox_bf16_proxy(int d_model, int d_ff, const uint16_t *w_cm, uint16_t *q16_out,
                            void *stream);

/*
 * prox_workspace_bytes -- bytes of device workspace prox_ffn_forward and
 * prox_proxy_state need for this shape and batch. The workspace must be
 * zero-filled once after allocation (cudaMemset to 0); the library leaves it
 * ready for the next call at the end of every call. One workspace serves one
 * stream at a time: calls that share it must not overlap on the device.
 */
size_t prox_workspace_bytes(int d_model, int d_ff, int batch);

/*
 * prox_ffn_forward -- Stage 1 then Stage 2 for `batch` tokens, each with its
 * own masks; tau_x and tau_s are per-layer scalars shared by all tokens
 * (blog, "Stage 1" and "Stage 2").
 *   x       : device, bf16 [batch][d_model].
 *   tau_x   : input threshold, finite and >= 0 (|x_i| >= tau_x is kept).
 *   tau_s   : channel threshold, finite and >= 0 (|s~_j| >= tau_s is kept).
 *   y       : device, fp32 [batch][d_model]; fully overwritten.
 *   mask_x  : device, uint8 [batch][d_model] (1 = kept input) or NULL.
 *   mask_s  : device, uint8 [batch][d_ff] (1 = kept channel) or NULL.
 *   idx_s   : device, int32 [batch][d_ff]; row t starts with the kept channels
 *             of token t in ascending order (the rest is left untouched) or NULL.
 *   count_s : device, int32 [batch], kept-channel count per token, or NULL.
 *   ws      : device workspace of at least prox_workspace_bytes(...) bytes.
 * Arithmetic: proxy products accumulate in fp32 from exact INT4 codes; exact
 * products read bf16 weights and accumulate in fp32; SiLU in fp32; y in fp32.
 * Errors: PROX_EINVAL (null required pointer, shape, negative or non-finite
 * threshold, misaligned pointer), PROX_ENOMEM (ws_bytes too small),
 * PROX_ECUDA (launch failure). Device-side wait timeouts are reported through
 * prox_last_device_status.
 */
prox_status prox_ffn_forward(const prox_layer *layer, const uint16_t *x, int batch,
                             float tau_x, float tau_s, float *y, uint8_t *mask_x,
                             uint8_t *mask_s, int32_t *idx_s, int32_t *count_s,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * prox_ffn_forward_static -- prox_ffn_forward without a caller workspace: the
 * library's own workspace is one file-scope device array of
 * PROX_STATIC_WORKSPACE_BYTES (2 MiB) per device, so the call allocates
 * nothing (no cudaMalloc/cudaFree, no allocating library). The Prox pages
 * have no counterpart of this entry point; it is for callers that cannot
 * allocate or hold device memory of their own, such as plain-C hosts with no
 * device allocator, or serving loops that must not call cudaMalloc/cudaFree
 * (both can synchronise the device) in steady state.
 *   Arguments, arithmetic and results as in prox_ffn_forward, minus ws.
 *   Limit: shapes with prox_workspace_bytes(d_model, d_ff, batch) above
 *     PROX_STATIC_WORKSPACE_BYTES are rejected with PROX_ENOMEM (for example
 *     d_model 4096 x d_ff 12288 fits at any batch; d_ff 262144 does not).
 *   Setup: the first call on a device looks the array up
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     outside any stream capture. Later calls only launch kernels.
 *   Sharing: every call on a device uses the same array, so calls must not
 *     overlap on the device (one stream, or ordered by the caller); two
 *     overlapping calls race on it.
 *   Timeouts: the array starts zero-filled (static device storage). When a
 *     bounded device-side wait gives up, the kernels set a bit of its status
 *     word and return early, and this call has still returned PROX_OK: read
 *     (and clear) that word with prox_static_last_device_status.
 * Errors: as prox_ffn_forward; PROX_ENOMEM for a shape over the limit;
 * PROX_ECUDA if the symbol lookup fails.
 */
#define PROX_STATIC_WORKSPACE_BYTES ((size_t)2 << 20)
prox_status prox_ffn_forward_static(const prox_layer *layer, const uint16_t *x, int batch,
                                    float tau_x, float tau_s, float *y, uint8_t *mask_x,
                                    uint8_t *mask_s, int32_t *idx_s, int32_t *count_s,
                                    void *stream);

/*
 * prox_static_last_device_status -- prox_last_device_status for the array of
 * prox_ffn_forward_static on the current device: copies its status word to
 * *flags_out (if not NULL) and clears it, after the work queued on `stream`
 * (synchronises `stream`). Returns PROX_ETIMEOUT if a bounded wait gave up
 * since the last read, else PROX_OK; PROX_ECUDA on a failed copy or lookup.
 * The first use on a device looks the array up like the forward does.
 */
prox_status prox_static_last_device_status(void *stream, uint32_t *flags_out);

/*
 * Layer stacks. The Prox pages define one FFN; a stack of FFN layers (as in
 * the stacked-layer benchmark) runs them pre-norm on an fp32 residual stream:
 *   x = bf16(RMSNorm(h)),  RMSNorm(h) = h / sqrt(mean(h^2) + eps) (unit gain),
 *   h <- h + FFN(x)        with FFN the Prox forward above.
 *
 * prox_rmsnorm_bf16 -- x_out = bf16 (round to nearest even) of
 *   h / sqrt(mean(h^2) + eps) per token, fp32 sum of squares in a fixed order.
 *   h : device, fp32 [batch][d_model];  x_out : device, bf16 [batch][d_model].
 *   Errors: PROX_EINVAL (null or misaligned pointer, bad shape, eps < 0 or
 *   not finite), PROX_EDEVICE, PROX_ECUDA.
 *
 * prox_ffn_block -- one layer of the stack: x_out = RMSNorm(h_in) as above,
 *   then h_out = h_in + FFN(x_out) with the Prox forward (Stage 2 adds its
 *   products onto a copy of h_in, so y is never stored). h_out may be h_in
 *   (in place). x_out (device, bf16 [batch][d_model]) is required: it is the
 *   FFN's input. Other arguments, workspace and errors as in
 *   prox_ffn_forward.
 */
prox_status prox_rmsnorm_bf16(int d_model, int batch, const float *h, float eps,
                              uint16_t *x_out, void *stream);
prox_status prox_ffn_block(const prox_layer *layer, const float *h_in, int batch,
                           float tau_x, float tau_s, float eps, float *h_out, uint16_t *x_out,
                           uint8_t *mask_x, uint8_t *mask_s, int32_t *idx_s, int32_t *count_s,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * prox_max_batch_per_pass -- tokens one Stage-1/Stage-2 pass handles for this
 * d_model (8 up to d_model 4096, 4 up to 8192, 0 beyond: unsupported).
 * prox_ffn_forward splits larger batches into passes by itself.
 */
int prox_max_batch_per_pass(int d_model);

/*
 * prox_set_stage2_engine -- which kernels run Stage 2 (process-wide; takes
 * effect at the next forward call, returns the previous setting, or -1 for
 * an unknown value, which changes nothing).
 *   PROX_ENGINE_AUTO (default): the tensor-core union engine for passes of 8
 *     tokens and, on layers of d_model >= 8192, of 4 tokens; the CUDA-core
 *     engine otherwise;
 *   PROX_ENGINE_SIMT: the CUDA-core engine always: per channel of the union,
 *     dot products of the kept rows with x on the CUDA cores;
 *   PROX_ENGINE_TC: the tensor-core engine for every pass of 4 or more
 *     tokens: the union's up/gate rows and the W_down rows are dense UMMA
 *     GEMMs over the pass's tokens (tcgen05, fp32 accumulators), each
 *     token's own channel mask applied to s, s carried as a bf16 hi + lo
 *     pair (relative error about 2^-16) into the down GEMM.
 * The pages give no kernel for batches beyond one token (blog, section
 * "Limitations"); both engines compute the per-token Stage 2 of the blog's
 * section "Stage 2" and differ only in summation order.
 */
#define PROX_ENGINE_AUTO 0
#define PROX_ENGINE_SIMT 1
#define PROX_ENGINE_TC 2
int prox_set_stage2_engine(int engine);

/*
 * prox_set_stage1_engine -- which kernels form the INT4 proxy products of
 * Stage 1 (process-wide, same values and return as prox_set_stage2_engine).
 *   PROX_ENGINE_AUTO (default) and PROX_ENGINE_TC: passes of 4 or 8 tokens
 *     with the INT4 proxy run the proxy products on the tensor cores
 *     (tcgen05 kind::i8: the codes as unsigned bytes, x_i * scale_i per token
 *     as a 27-bit fixed-point value in four signed 8-bit digits, int32
 *     accumulation, so the CTA's sums are exact up to that fixed point);
 *     smaller passes and the bf16 proxy use the CUDA cores;
 *   PROX_ENGINE_SIMT: the CUDA cores always.
 * Masks, lists and the proxy state are formed the same way after either.
 */
int prox_set_stage1_engine(int engine);

/*
 * prox_ffn_stage1 / prox_ffn_stage2 -- the two phases of prox_ffn_forward,
 * callable separately (for instance to time or inspect Stage 1 alone).
 * prox_ffn_forward(..) with batch <= prox_max_batch_per_pass(d_model) is
 * exactly prox_ffn_stage1 followed by prox_ffn_stage2 on the same workspace.
 *   prox_ffn_stage1: masks (as in prox_ffn_forward) plus the kept-channel
 *     lists, left in `ws`; clears y_clear (device, fp32 [batch][d_model],
 *     may be NULL when Stage 2 will not run).
 *   prox_ffn_stage2: exact Stage 2 from the lists the immediately preceding
 *     prox_ffn_stage1 call on the same `ws`, same x and batch, left there;
 *     accumulates into y, which that Stage-1 call cleared; writes idx_s and
 *     count_s (either may be NULL).
 * Both require 0 <= batch <= prox_max_batch_per_pass(d_model) (else
 * PROX_EINVAL); other arguments and errors as in prox_ffn_forward.
 */
prox_status prox_ffn_stage1(const prox_layer *layer, const uint16_t *x, int batch,
                            float tau_x, float tau_s, float *y_clear, uint8_t *mask_x,
                            uint8_t *mask_s, void *ws, size_t ws_bytes, void *stream);
prox_status prox_ffn_stage2(const prox_layer *layer, const uint16_t *x, int batch, float *y,
                            int32_t *idx_s, int32_t *count_s, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * prox_proxy_state -- Stage 1 alone: writes the proxy intermediate state
 * s~ = u~ (.) SiLU(g~) (blog, "Stage 1") for every channel of every token.
 *   s_out  : device, fp32 [batch][d_ff].
 *   mask_x : device, uint8 [batch][d_model] or NULL.
 * Other arguments as in prox_ffn_forward.
 */
prox_status prox_proxy_state(const prox_layer *layer, const uint16_t *x, int batch,
                             float tau_x, float *s_out, uint8_t *mask_x, void *ws,
                             size_t ws_bytes, void *stream);

/*
 * prox_calibrate_workspace_bytes -- device workspace prox_calibrate needs.
 */
size_t prox_calibrate_workspace_bytes(int d_model, int d_ff, int n_cal);

/*
 * prox_calibrate -- per-layer thresholds from calibration vectors (blog,
 * "Stage 1": offline per-layer thresholds; "Evidence": thresholds taken from
 * calibration activations, layer by layer).
 * Reading: tau is the exact order statistic of the pooled magnitudes. With the
 * n pooled values sorted ascending v[0..n-1] and
 * rank = floor((1 - keep) * n) (IEEE double, clamped to [0, n-1]):
 *   tau_x = v[rank] over |x| of all n_cal x d_model calibration coordinates;
 *   tau_s = v[rank] over |s~| of all n_cal x d_ff channels, with s~ computed
 *           by Stage 1 at the tau_x just found.
 *   x_cal     : device, bf16 [n_cal][d_model]; n_cal >= 1.
 *   keep_x, keep_s : kept fractions in [0, 1].
 *   tau_x_out, tau_s_out : HOST pointers, written before the call returns.
 *   ws        : device, >= prox_calibrate_workspace_bytes(...) bytes, zero-filled
 *               once after allocation (left ready for reuse).
 * The only call that synchronises `stream`.
 */
prox_status prox_calibrate(const prox_layer *layer, const uint16_t *x_cal, int n_cal,
                           double keep_x, double keep_s, float *tau_x_out,
                           float *tau_s_out, void *ws, size_t ws_bytes, void *stream);

/*
 * prox_calibrate_histogram -- prox_calibrate with the pages' bounded
 * calibration (blog, "Evidence": at most 200,000 activation samples and a
 * 4,096-bin histogram per layer) instead of the exact order statistic:
 *   samples: every k-th pooled magnitude, k = ceil(n / max_samples), in pooled
 *            order (x_cal row by row; s~ token by token, channel by channel);
 *   bins:    `bins` equal bins of width w = m / bins over [0, m], m the
 *            largest sample; a sample s falls in bin trunc(fp32(s / w)), m in
 *            the top bin;
 *   tau:     fp32(b * w), the lower edge of the bin holding the sample of rank
 *            floor((1 - keep) * n_samples), so at least the asked-for share of
 *            samples is kept.
 *   max_samples >= 1; bins a multiple of 1024 in [1024, 65536] (the pages:
 *   200000 and 4096). Workspace as prox_calibrate. Synchronises `stream`.
 * Errors: as prox_calibrate; PROX_EINVAL for max_samples or bins outside range.
 */
prox_status prox_calibrate_histogram(const prox_layer *layer, const uint16_t *x_cal, int n_cal,
                                     double keep_x, double keep_s, long max_samples, int bins,
                                     float *tau_x_out, float *tau_s_out, void *ws,
                                     size_t ws_bytes, void *stream);

/*
 * prox_allocate -- split a target effective sparsity between the stages
 * (blog, "Compute budget"): C = 2 alpha (1 - s1) + 3 (1 - s2) and
 * e = 1 - C/3 = s2 - 2 alpha (1 - s1) / 3.
 * Reading of the allocation rule: anchor s2 at s2_anchor and solve for s1; if
 * s1 falls outside [0, s1_max], clamp it and solve for s2. The blog's case
 * e = 0.7, alpha = 1/3, s1_max = 0.7, anchor 0.7 gives s1 = 0.7, s2 ~= 0.7667.
 * Host only; s1_out and s2_out are host pointers.
 * Errors: PROX_EINVAL on null outputs, alpha <= 0, or e, s1_max, s2_anchor
 * outside [0, 1].
 */
prox_status prox_allocate(double e, double alpha, double s1_max, double s2_anchor,
                          double *s1_out, double *s2_out);

/*
 * prox_last_device_status -- reads and clears the device status word in a
 * forward workspace (synchronises `stream`). Returns PROX_ETIMEOUT if a
 * bounded device-side wait gave up since the last read, PROX_OK otherwise.
 * *flags_out (host, may be NULL) receives the raw status bits.
 */
prox_status prox_last_device_status(void *ws, size_t ws_bytes, void *stream,
                                    uint32_t *flags_out);

/* Static English description of a status code. */
const char *prox_status_str(prox_status status);

#ifdef __cplusplus
}
#endif

#endif /* PROX_H */
