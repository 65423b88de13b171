/*
 * qmoe.h -- C ABI of the B200 (sm_100a) weight-only-quantized MoE forward.
 *
 * The operator is the QMoE node defined on the "QMoE" operator page
 * (graiphic.io: inputs input, router_probs, fc1/fc2/fc3 expert weights,
 * scales and biases; attributes activation_alpha, activation_beta,
 * activation_type, block_size, expert_weight_bits, k,
 * normalize_routing_weights, swiglu_fusion, swiglu_limit, use_sparse_mixer),
 * with the module lifecycle of "ClikaRT::nn::QMoEWoQ" (make(), set_weights(),
 * forward(), ~QMoEWoQ()). Expert weights stay packed as 4- or 8-bit integers
 * and are decoded block by block inside the GEMM dot ("ClikaRT::nn::QMoEWoQ",
 * class description); no dense copy of any weight is ever made.
 *
 * Conventions for every call below
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, and are
 *     borrowed for the duration of the call (or of the stream work it
 *     enqueues, for qmoe_forward).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.
 *   - No call throws; each returns a qmoe_status. The handle keeps the text of
 *     its last error (qmoe_last_error).
 *   - Packed weight layout is the QMoE page's: a [E, N, K/pack] uint8 stack,
 *     pack = 8/expert_weight_bits along K. Codes are unsigned with an implicit
 *     zero point 2^(bits-1); with 4 bits the even k of a pair sits in the low
 *     nibble. (The page gives no zero-point input; this is the reading taken.)
 */
#ifndef QMOE_H
#define QMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QMOE_API __attribute__((visibility("default")))
#else
#define QMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qmoe_status {
    QMOE_OK = 0,
    /* Shape, dtype or geometry mismatch; a bias without its declared slot;
     * block_size not a power of two >= 16 or not dividing H and I; bits not
     * 4 or 8; k outside [1, E]; a NULL required pointer; a workspace too small
     * or not 256-byte aligned ("ClikaRT::nn::QMoEWoQ", set_weights() and
     * forward(): Error on geometry or shape mismatch). */
    QMOE_INVALID_ARGUMENT = 1,
    /* forward() before set_weights() bound the required slots (the "still-fake
     * slot" error of "ClikaRT::nn::QMoEWoQ", forward() and initialize_impl()). */
    QMOE_NOT_BOUND = 2,
    /* Valid per the pages but not built here: use_sparse_mixer, E > 256,
     * H or I not a multiple of 64. */
    QMOE_UNSUPPORTED = 3,
    QMOE_CUDA_ERROR = 4,
    /* A bounded device-side wait gave up (see qmoe_read_device_status). */
    QMOE_TIMEOUT = 5,
    QMOE_OUT_OF_MEMORY = 6
} qmoe_status;

/* activation_type, in the order the QMoE page lists them. */
enum {
    QMOE_ACT_RELU = 0,
    QMOE_ACT_GELU = 1, /* erf form, or the tanh form with gelu_mode QMOE_GELU_TANH */
    QMOE_ACT_SILU = 2,
    QMOE_ACT_SWIGLU = 3,
    QMOE_ACT_IDENTITY = 4
};

/* dtypes; E8M0 (a power-of-two exponent byte, value 2^(x - 127)) is a
 * scale dtype of MXFP4 weights only. */
enum { QMOE_DTYPE_F32 = 0, QMOE_DTYPE_BF16 = 1, QMOE_DTYPE_E8M0 = 2 };

/* weight_format. INT: unsigned integer codes with the implicit zero point
 * 2^(bits-1). MXFP4 (the block format of the QMoEWoQ page's gpt-oss
 * checkpoint, read as the OCP microscaling FP4 format): each 4-bit code is
 * e2m1 -- sign, two exponent bits, one mantissa bit, magnitudes 0, 0.5, 1,
 * 1.5, 2, 3, 4, 6 -- packed two per byte like int4 (even k in the low
 * nibble), with one E8M0 scale per 32 codes along K; requires
 * expert_weight_bits 4, block_size 32 and scale_dtype E8M0. The activations
 * stay floating point either way. */
enum { QMOE_WEIGHTS_INT = 0, QMOE_WEIGHTS_MXFP4 = 1 };

/* compute_mode ("ClikaRT::nn::QMoEWoQ" page, class description: a packed
 * block weight on the int8 block tier rounds the activation to per-block int8
 * before the dot; the pages give no rounding rule). FLOAT: the activations
 * stay floating point. INT8_BLOCK: every expert input row -- x (or the
 * router-weighted row, rounded to act_dtype) for FC1, h rounded to act_dtype
 * for FC2 -- is cut into the weight's K blocks and rounded per block with
 * s = absmax / 127 and q = clamp(rint(v / s), -127, 127), ties to even,
 * decided in fp32 (s = 0, q = 0 for an all-zero block); each weight row then
 * sums s_w * s * (integer dot of (code - zero point) and q) over its blocks.
 * Requires weight_format INT and block_size >= 64 (4-bit codes) or >= 32
 * (8-bit codes); runs on path 4 for every T and both act dtypes. */
enum { QMOE_COMPUTE_FLOAT = 0, QMOE_COMPUTE_INT8_BLOCK = 1 };

/*
 * Operator attributes ("QMoE" page attribute list; "ClikaRT::nn::QMoEWoQ",
 * make(): the four counts and the bias flags).
 *
 * Gating: the FFN is gated (h = act(gate) * up, or swiglu) when
 * swiglu_fusion is 1 (rows 2i = gate, 2i+1 = up) or 2 (rows [0, I) = gate,
 * [I, 2I) = up), or when has_fc3 is set with swiglu_fusion 0 (fc1 = gate,
 * fc3 = up). Otherwise h = act(fc1 x + b1) and swiglu is invalid.
 *
 * swiglu: g' = min(g, L), u' = clamp(u, -L, L),
 *         h = (u' + beta) * g' * sigmoid(alpha * g').
 * activation_alpha == 0 reads as 1 (the page's default 0 would not be
 * SwiGLU); swiglu_limit <= 0 or non-finite means no clamp (the page states the
 * limit is infinite when not provided).
 */
typedef struct qmoe_config {
    int64_t num_experts;          /* E, 1..256 */
    int64_t hidden_size;          /* H, multiple of 64 */
    int64_t inter_size;           /* I, multiple of 64 */
    int64_t k;                    /* experts per token, 1..E */
    int32_t expert_weight_bits;   /* 4 or 8 */
    int32_t block_size;           /* 0 = one scale per output row; else power of two >= 16 */
    int32_t activation_type;      /* QMOE_ACT_* */
    int32_t swiglu_fusion;        /* 0, 1, 2 */
    float activation_alpha;
    float activation_beta;
    float swiglu_limit;
    int32_t normalize_routing_weights; /* renormalise the k weights to sum to 1 */
    int32_t act_dtype;            /* dtype of x, router_logits, shared_output, biases and y */
    int32_t scale_dtype;          /* dtype of fc1/fc2/fc3 scales */
    int32_t has_fc1_bias;
    int32_t has_fc2_bias;
    int32_t has_fc3;
    int32_t has_fc3_bias;
    int32_t use_sparse_mixer;     /* must be 0 */
    int32_t reserved;             /* must be 0 */
    /* Routing options the "MoE" page names (n_group, topk_group,
     * routed_scaling_factor, apply_router_weight_on_input) without formulas;
     * readings:
     *   grouped top-k -- the E experts form n_group consecutive groups of
     *     E / n_group; a group's score is the largest raw logit among its
     *     experts; the topk_group best groups are kept (ties to the lower group
     *     id) and the k experts are the top-k by logit among their experts.
     *     n_group 0 or 1: no grouping. Otherwise E % n_group == 0,
     *     n_group <= 32, 1 <= topk_group <= n_group and
     *     k <= topk_group * E / n_group.
     *   routed_scaling_factor -- multiplies the router-weighted sum of the
     *     expert outputs (not the shared output); 0 reads as 1.
     *   apply_router_weight_on_input -- 1: the router weight scales the
     *     expert's input row (rounded to the activation dtype) instead of its
     *     output; the combine then sums the expert outputs unweighted. */
    int32_t n_group;
    int32_t topk_group;
    float routed_scaling_factor;
    int32_t apply_router_weight_on_input;
    int32_t weight_format;        /* QMOE_WEIGHTS_* */
    int32_t compute_mode;         /* QMOE_COMPUTE_* */
    /* Options the "MoE" page names without formulas; readings:
     *   expert_output_scale -- multiplies every expert's output (its fc2 bias
     *     included) before the router weighting; 0 reads as 1; finite, >= 0.
     *   gelu_mode -- QMOE_GELU_ERF (default) or QMOE_GELU_TANH, the form of
     *     activation_type GELU (plain or gated): erf, or the tanh form
     *     0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3))). */
    float expert_output_scale;
    int32_t gelu_mode;
} qmoe_config;

enum { QMOE_GELU_ERF = 0, QMOE_GELU_TANH = 1 };

typedef struct qmoe_handle qmoe_handle;

/*
 * qmoe_create -- "ClikaRT::nn::QMoEWoQ", make(): validate the attributes and
 * declare storage-free weight slots. Allocates host memory only; touches no
 * GPU. On success *out owns a handle that qmoe_destroy releases.
 */
QMOE_API qmoe_status qmoe_create(const qmoe_config* cfg, qmoe_handle** out);

/*
 * qmoe_set_weights -- "ClikaRT::nn::QMoEWoQ", set_weights() followed by the
 * one-time pack of initialize_impl().
 *
 *   fc1_w  [E, N1, H*bits/8] uint8, N1 = 2I if swiglu_fusion is 1 or 2, else I
 *   fc1_s  [E, N1, H/block_size] or [E, N1] (block_size 0), scale_dtype
 *   fc1_b  [E, N1] act_dtype; required iff has_fc1_bias, else must be NULL
 *   fc2_w  [E, H, I*bits/8] uint8
 *   fc2_s  [E, H, I/block_size] or [E, H]
 *   fc2_b  [E, H]; required iff has_fc2_bias
 *   fc3_w  [E, I, H*bits/8], fc3_s like fc1_s with I rows; required iff has_fc3
 *   fc3_b  [E, I]; required iff has_fc3_bias
 *
 * All pointers are device pointers; scales and biases aligned to their
 * element size (QMOE_INVALID_ARGUMENT otherwise), codes at any address. The
 * call re-lays the packed bytes into the
 * kernels' tile order in handle-owned device memory of the same size (the
 * weights stay quantized; this copy is the one resident copy), waits for that
 * work on `stream`, and returns; the caller may then free its buffers. A
 * second call drops the previous pack and packs again.
 */
QMOE_API qmoe_status qmoe_set_weights(qmoe_handle* h,
                             const void* fc1_w, const void* fc1_s, const void* fc1_b,
                             const void* fc2_w, const void* fc2_s, const void* fc2_b,
                             const void* fc3_w, const void* fc3_s, const void* fc3_b,
                             void* stream);

/*
 * qmoe_set_score_correction_bias -- the e_score_correction_bias tensor of
 * "ClikaRT::nn::QMoEWoQ" / the QMoEWoQ Python page, set_weights(); the pages
 * give no formula. Reading: the bias moves the expert selection only. Every
 * forward then ranks experts (and, with grouped top-k, groups by their
 * largest key) by the fp32 sum logit + bias[e], one single-precision
 * addition, ties to the lower id; the router weights stay the softmax of the
 * unbiased logits over all E, restricted to the selection.
 *
 *   bias  [E] fp32, a DEVICE pointer aligned to 4 bytes, or NULL to clear
 *
 * The values are copied into handle-owned device memory (the call waits for
 * the copy on `stream`); the caller may free its buffer afterwards. A NaN
 * key reads as -inf. QMOE_INVALID_ARGUMENT for a misaligned pointer.
 */
QMOE_API qmoe_status qmoe_set_score_correction_bias(qmoe_handle* h, const void* bias, void* stream);

/*
 * qmoe_workspace_size -- bytes of device scratch that qmoe_forward needs for
 * T tokens (routing lists, permutation, hidden activations, partial sums).
 * Returns 0 for a NULL handle or T < 0.
 */
QMOE_API size_t qmoe_workspace_size(const qmoe_handle* h, int64_t T);

/*
 * qmoe_forward -- "ClikaRT::nn::QMoEWoQ", forward(): one MoE step.
 *
 *   x              [T, H] act_dtype, 16-byte aligned
 *   router_logits  [T, E] act_dtype (logits; softmax is applied inside),
 *                  aligned to its element size
 *   shared_output  [T, H] act_dtype or NULL (folded into the combine),
 *                  16-byte aligned
 *   y              [T, H] act_dtype (written), 16-byte aligned
 *   workspace      >= qmoe_workspace_size(h, T) bytes, 256-byte aligned,
 *                  owned by the caller; contents on entry are ignored
 *
 * For T > 0 a NULL required pointer or a misaligned one is
 * QMOE_INVALID_ARGUMENT, checked before the handle's binding
 * (QMOE_NOT_BOUND).
 *
 * Enqueues all work on `stream` and returns without waiting; it never
 * synchronises the host. The handle is only read, so concurrent calls on
 * different streams with different workspaces are safe. T == 0 is a no-op.
 * A 3-D [B, S, H] input is passed as T = B*S.
 */
QMOE_API qmoe_status qmoe_forward(const qmoe_handle* h, int64_t T, const void* x, const void* router_logits,
                         const void* shared_output, void* y, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * qmoe_forward_profiled -- qmoe_forward that also records CUDA events on
 * `stream` around its kernels: events[i] just before launch i and
 * events[n_events - 1] after the last launch. `events` holds cudaEvent_t
 * handles created by the caller with timing enabled; n_events must equal
 * qmoe_launches_for(h, T) + 1. The kernels and their order are the same as
 * qmoe_forward's, so elapsed times between consecutive events are the
 * per-kernel device times of a normal forward.
 */
QMOE_API qmoe_status qmoe_forward_profiled(const qmoe_handle* h, int64_t T, const void* x,
                                           const void* router_logits, const void* shared_output,
                                           void* y, void* workspace, size_t workspace_bytes,
                                           void* stream, void* const* events, int32_t n_events);

/*
 * qmoe_debug_routing -- copy the routing and permutation of the last forward
 * that used `workspace` into caller DEVICE buffers (test support; enqueued on
 * `stream`). Any output pointer may be NULL to skip it.
 *   topk_idx [T, k] int32   selected experts, (logit desc, id asc) order
 *   topk_w   [T, k] float   router weights
 *   offsets  [E + 1] int32  segment starts; offsets[E] = T*k
 *   perm_tok [T*k] int32    token of each permuted row
 *   inv      [T, k] int32   permuted row of (token, slot)
 */
QMOE_API qmoe_status qmoe_debug_routing(const qmoe_handle* h, int64_t T, const void* workspace,
                               int32_t* topk_idx, float* topk_w, int32_t* offsets,
                               int32_t* perm_tok, int32_t* inv, void* stream);

/*
 * qmoe_debug_hidden -- copy the hidden activations h [T*k, I] (permuted row
 * order, act_dtype) of the last forward that used `workspace` into a caller
 * DEVICE buffer (test support; enqueued on `stream`).
 */
QMOE_API qmoe_status qmoe_debug_hidden(const qmoe_handle* h, int64_t T, const void* workspace,
                              void* hidden, void* stream);

/*
 * qmoe_read_device_status -- wait for `stream`, then read the device-side
 * status word of `workspace` (QMOE_OK, QMOE_TIMEOUT when a bounded device
 * wait gave up in the last forward that used it, or QMOE_INVALID_ARGUMENT
 * when qmoe_ep_expert_rows met an expert id outside its handle's range).
 */
QMOE_API qmoe_status qmoe_read_device_status(const qmoe_handle* h, const void* workspace, void* stream);

/*
 * qmoe_forward_noalloc -- qmoe_forward without a caller workspace. (The
 * operator pages have no counterpart; this is a deployment convenience.)
 *
 * For callers that cannot allocate device memory where they run the operator
 * -- a plugin whose host framework owns all device memory and passes in only
 * the input and output buffers, or a serving loop that must not allocate while
 * it handles a request. The scratch is one fixed library-owned device array of
 * qmoe_noalloc_scratch_bytes() bytes (8 MiB), which every GPU that loads the
 * library holds until the process exits. Arguments are qmoe_forward's minus
 * the workspace; a T whose qmoe_workspace_size exceeds the array returns
 * QMOE_INVALID_ARGUMENT with the sizes in qmoe_last_error. Nothing is allocated
 * or freed.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture (a first call on a capturing stream returns
 * QMOE_INVALID_ARGUMENT). All calls share the one array, which keeps the
 * last call's contents: calls whose GPU work can overlap (other streams,
 * other host threads) race on it and must be serialised by the caller.
 */
QMOE_API qmoe_status qmoe_forward_noalloc(const qmoe_handle* h, int64_t T, const void* x,
                                          const void* router_logits, const void* shared_output,
                                          void* y, void* stream);

/* Size in bytes of the fixed scratch array behind qmoe_forward_noalloc. */
QMOE_API size_t qmoe_noalloc_scratch_bytes(void);

/*
 * qmoe_noalloc_read_device_status -- qmoe_read_device_status for the forward
 * run by qmoe_forward_noalloc on the current device: wait for `stream`, then
 * read the device status word in the fixed scratch array (QMOE_OK, or
 * QMOE_TIMEOUT when a bounded device wait of the last no-alloc forward on
 * this device gave up). QMOE_INVALID_ARGUMENT if no no-alloc forward has run
 * on the current device. (No counterpart on the pages.)
 */
QMOE_API qmoe_status qmoe_noalloc_read_device_status(const qmoe_handle* h, void* stream);

/*
 * Expert parallel: the forward split at its two exchange points, for experts
 * spread over ranks (each rank holds a contiguous range of experts in its own
 * handle, every rank routes its own tokens). The pages fix no parallelism;
 * the steps are those of qmoe_forward ("ClikaRT::nn::QMoEWoQ", forward();
 * the "MoE" page's routed combine) with the rows moved between ranks by the
 * caller (an all-to-all) after dispatch and again after the expert rows.
 *
 * qmoe_ep_dispatch -- on the token owner, with a handle of the full expert
 * set (weights need not be bound: only the routing attributes and the score
 * correction bias are used): route T tokens, sort their T*k routes by expert
 * (stable, token order inside an expert) and write
 *   rows       [T*k, H] act_dtype  x's row of every route, in that order
 *                                  (scaled by the router weight and rounded
 *                                  to act_dtype with apply_router_weight_on_input)
 *   row_expert [T*k] int32         the global expert id of each row
 *   offsets    [E+1] int32         rows of expert e are offsets[e] .. offsets[e+1]
 *   state      qmoe_ep_state_bytes(h, T) bytes: the routing, for qmoe_ep_combine
 * All DEVICE pointers; x and rows 16-byte aligned, state 256-byte aligned.
 * The rows destined to one rank are one contiguous range (its experts'
 * offsets). Enqueued on `stream`; T = 0 is a no-op.
 */
QMOE_API size_t qmoe_ep_state_bytes(const qmoe_handle* h, int64_t T);
QMOE_API qmoe_status qmoe_ep_dispatch(const qmoe_handle* h, int64_t T, const void* x, const void* router_logits,
                                      void* rows, int32_t* row_expert, int32_t* offsets, void* state,
                                      size_t state_bytes, void* stream);

/*
 * qmoe_ep_expert_rows -- on the expert owner, with a handle holding experts
 * expert_base .. expert_base + E_h - 1 (its num_experts = E_h, weights
 * bound): for R rows of any order, out[r] [H] fp32 = FC2(act(FC1(rows[r])))
 * + fc2 bias of expert row_expert[r] - expert_base (no router weight, no
 * scaling factor: the token owner's combine applies them). The handle's
 * routing attributes (k, normalisation, scaling, router weight on input) are
 * not used. rows [R, H] act_dtype and out 16-byte aligned; workspace of
 * qmoe_ep_rows_workspace_size(h, R) bytes, 256-byte aligned. An id outside
 * the handle's range is not an index: the row is computed as expert 0 and
 * the workspace status word reads QMOE_INVALID_ARGUMENT
 * (qmoe_read_device_status). R = 0 is a no-op.
 */
QMOE_API size_t qmoe_ep_rows_workspace_size(const qmoe_handle* h, int64_t R);
QMOE_API qmoe_status qmoe_ep_expert_rows(const qmoe_handle* h, int64_t R, const void* rows,
                                         const int32_t* row_expert, int32_t expert_base, float* out,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * qmoe_ep_combine -- on the token owner, after the expert outputs came back
 * in dispatch order: y[t] = s * sum_j w[t, j] * expert_out[row of (t, j)] +
 * shared_output[t], rounded once to act_dtype (s = routed_scaling_factor x
 * expert_output_scale; w = 1 with apply_router_weight_on_input). expert_out
 * [T*k, H] fp32, the state of the matching qmoe_ep_dispatch; same handle.
 */
QMOE_API qmoe_status qmoe_ep_combine(const qmoe_handle* h, int64_t T, const float* expert_out, const void* state,
                                     const void* shared_output, void* y, void* stream);

/* qmoe_destroy -- "ClikaRT::nn::QMoEWoQ", ~QMoEWoQ(): release the packed
 * weights and the handle. NULL is a no-op. */
QMOE_API void qmoe_destroy(qmoe_handle* h);

/* Static text for a status code. */
QMOE_API const char* qmoe_status_string(qmoe_status s);

/* Text of the handle's last error ("" if none); valid until the next call on
 * the handle. */
QMOE_API const char* qmoe_last_error(const qmoe_handle* h);

/*
 * qmoe_quantize_act_i8 -- the int8 block tier's activation rounding as a
 * standalone operation (see compute_mode): rows x [rows, K] of dtype
 * (QMOE_DTYPE_F32 or QMOE_DTYPE_BF16) to codes q [rows, K] int8 in k order
 * and scales [rows, K / block_size] fp32, on `stream` (asynchronous). All
 * pointers are DEVICE pointers owned by the caller; x 16-byte aligned, q and
 * scales 4-byte aligned. block_size is a power of two >= 16 dividing K.
 * rows == 0 is a no-op. QMOE_INVALID_ARGUMENT for a bad size, dtype or
 * alignment; QMOE_CUDA_ERROR if the launch fails.
 */
QMOE_API qmoe_status qmoe_quantize_act_i8(const void* x, int32_t dtype, int64_t rows, int64_t K,
                                          int32_t block_size, int8_t* q, float* scales, void* stream);

/* Tunable options (qmoe_set_option). QMOE_OPT_PATH selects the expert-FFN
 * kernels for bf16 activations: -1 (default) chooses by shape, 1 forces the
 * weight-streaming mma.sync kernels, 2 the tcgen05 grouped GEMM, 3 the
 * tcgen05 streaming decode kernels (falls back to 1 for shapes they do not
 * cover: more than 32 rows per expert, K not a multiple of 128, or a K range
 * whose resident activations exceed 128 KB). fp32 activations always take
 * the fp32 path (0). Under compute_mode INT8_BLOCK the option chooses within
 * the tier: 1 (or 3) forces the streaming integer kernels (path 4), 2 the
 * tcgen05 integer GEMM (path 5; falls back to 4 for fp32 activations or
 * blocks of fewer than 32 codes); by default path 5 is taken for blocks of
 * 128 or more codes beyond 32 rows per expert, path 4 otherwise. */
enum { QMOE_OPT_PATH = 1 };

/* QMOE_OPT_WAIT_LIMIT_NS: the limit, in nanoseconds, of every bounded
 * device-side wait of the tcgen05 kernels (paths 2 and 3): 1e5 .. 6e10,
 * default 2e9. A wait that runs out sets QMOE_TIMEOUT in the workspace status
 * word (qmoe_read_device_status); every role of the kernel then leaves its
 * loop, the CTA frees its tensor memory, and the call's later kernels still
 * run (their results are then undefined).
 * QMOE_OPT_TEST_WITHHOLD (test support for that failure path; 0 or 1): with
 * 1, the MMA-issuing warp of each path-2 CTA never announces its first work
 * item's accumulator, so the epilogue's wait runs out after the limit. No
 * memory is touched out of place and no copy is left in flight; the next
 * forward with the option back at 0 is a normal one. */
enum { QMOE_OPT_WAIT_LIMIT_NS = 2, QMOE_OPT_TEST_WITHHOLD = 3 };

/* QMOE_OPT_PDL (0 or 1, default 1): launch the weight-streaming kernels of
 * path 1 and the combine as programmatic dependents of the kernel before
 * them, so each starts streaming its weights while the previous one drains;
 * 0 launches every kernel in plain stream order. Results are identical. */
enum { QMOE_OPT_PDL = 4 };

/* QMOE_OPT_DECODE_TILES (0, 1, 2 or 4; default 0): 8-token tiles per pass of
 * the weight-streaming kernels (paths 1 and 4); 0 chooses by the average rows
 * per expert. Fewer are taken where the staged activation rows of a pass
 * would not fit two CTAs per SM. An expert segment longer than one pass
 * streams its weights once per pass. Results agree with the oracle for every
 * value. */
enum { QMOE_OPT_DECODE_TILES = 5 };

/* qmoe_set_option -- set a tunable option on the handle. QMOE_INVALID_ARGUMENT
 * for an unknown option or value. Not thread-safe against concurrent
 * qmoe_forward calls on the same handle. */
QMOE_API qmoe_status qmoe_set_option(qmoe_handle* h, int32_t option, int64_t value);

/* The forward path qmoe_forward takes for T tokens: 0 = fp32 SIMT path,
 * 1 = weight-streaming decode path (mma.sync), 2 = tcgen05 grouped GEMM,
 * 3 = tcgen05 streaming decode, 4 = int8 block tier (weight-streaming
 * integer mma.sync), 5 = int8 block tier on the tcgen05 integer GEMM
 * (kind::i8, int32 accumulators in tensor memory folded per K block).
 * -1 for a NULL handle. */
QMOE_API int32_t qmoe_path_for(const qmoe_handle* h, int64_t T);

/* Number of kernel launches qmoe_forward enqueues for T tokens: routing and
 * permutation (one launch for T <= 64, two above), the row gather (tensor-core
 * paths, and apply_router_weight_on_input), the int8 rounding of FC1's and
 * FC2's input rows (int8 block tier), FC1, FC2 and the combine. 0 for T = 0. */
QMOE_API int32_t qmoe_launches_for(const qmoe_handle* h, int64_t T);

/* Token-tile width (the MMA N dimension, rows of one expert per work item)
 * of the tensor-core paths for T tokens: 16..128 run the 128-wide tcgen05
 * kernel with the decoded weights in TMEM, 256 the wide kernel with them in
 * shared memory; 16 or 32 on path 3; 16..64 on path 5. 0 on paths 0, 1 and
 * 4, -1 for a NULL
 * handle or T < 0. No counterpart on the pages: it only reports the plan. */
QMOE_API int32_t qmoe_token_tile_for(const qmoe_handle* h, int64_t T);

#ifdef __cplusplus
}
#endif

#endif /* QMOE_H */
