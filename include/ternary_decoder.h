/*
 * ternary_decoder.h — C ABI of the B200 ternary-weight linear layer.
 *
 * The layer is the 1.58-bit ("BitNet") projection of the VibeVoice-ASR-BitNet
 * LM decoder: every projection matrix W [N x K] is ternarised per tensor with
 * s = 1/mean|W| to codes in {-1, 0, +1} ("VibeVoice-ASR-BitNet-ONNX" model
 * page, "Quantization" table, row "LM projections (196 mats)"), activations
 * are quantised per token to int8 by absmax, multiplied with the codes in
 * integer arithmetic (ternary weights turn the multiply into add/subtract:
 * xujun.org article, heterogeneous-quantisation section) and rescaled by
 * absmax/127 and 1/s.  A Qwen2.5-1.5B-shaped decoder has 28 layers x 7
 * projections = 196 such matrices (the same Quantization table).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Matrices are row-major.  W is [N x K] (PyTorch Linear layout), x is
 *    [M x K], y = x W^T is [M x N].  Indices and sizes are int64_t.
 *  - Unless stated otherwise every pointer is a DEVICE pointer to memory the
 *    caller allocated and owns; the library allocates nothing that outlives a
 *    call.  Scratch memory is passed in as `ws` of `ws_bytes`, sized by the
 *    matching *_workspace_bytes query.
 *  - Work is enqueued on the caller's stream and the call returns without
 *    waiting.  Argument errors are detected on the host and returned at once;
 *    errors found by a kernel (non-finite weights, a timed-out wait) are
 *    recorded in a per-device error word and returned by tw_check().
 *  - Every device pointer must be 16-byte aligned.  K must be a positive
 *    multiple of 128 (the pages' ternary file format packs 128 weights per
 *    unit: "The Paper Says ARM Support" post, "Postscript two").
 *  - Return value: TW_OK or one of the TW_ERR_* codes; tw_last_error() gives
 *    a message for the last failing call on the calling host thread.
 *
 * Packed code layout (this library's own design)
 * ----------------------------------------------
 * Codes are stored as c + 1 in {0, 1, 2} in two bits (pattern 3 is invalid),
 * sixteen consecutive-k codes of one row per 32-bit word: the code of
 * k0 + 4*s + b sits at bit 8*b + 2*s, so (word >> 2*s) & 0x03030303 yields
 * four consecutive codes as bytes.  Rows are grouped in blocks of 16 (N is
 * padded up to a multiple of 16 with code 0); a tile is 16 rows x 128 k =
 * 512 bytes; tiles are stored row-block-major (all K/128 tiles of rows
 * 16r..16r+15 are contiguous).  Inside a tile, 32-bit word 4*l + j (l = 4g + t,
 * g in 0..7, t in 0..3, j in 0..3) holds row g + 8*(j & 1) and
 * k = 64*(j >> 1) + 16*t .. +15, so each 16-byte lane slot of a tile is what
 * one lane of a warp needs for two m16n8k32 integer MMA fragments.
 */
#ifndef TERNARY_DECODER_H
#define TERNARY_DECODER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TW_API __attribute__((visibility("default")))
#else
#define TW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream; identical to cudaStream_t.  NULL is the legacy default. */
typedef struct CUstream_st *tw_stream_t;

enum {
    TW_OK = 0,
    TW_ERR_NULL = 1,       /* a required pointer is NULL                    */
    TW_ERR_SHAPE = 2,      /* N < 1, M < 1, K < 1, K % 128 != 0, or too big */
    TW_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned              */
    TW_ERR_BUFSIZE = 4,    /* a buffer or workspace is smaller than needed  */
    TW_ERR_NONFINITE = 5,  /* W holds Inf or NaN (reported by tw_check)     */
    TW_ERR_CUDA = 6,       /* a CUDA runtime call failed                    */
    TW_ERR_TIMEOUT = 7,    /* a bounded device-side wait expired (tw_check) */
    TW_ERR_CORRUPT = 8,    /* a table or packed buffer is malformed         */
    TW_ERR_UNSUPPORTED = 9 /* no sm_100 device, or a mode not built         */
};

/* Bytes of packed codes for an [N x K] matrix: ceil(N/16)*16 * K / 4. */
TW_API size_t tw_packed_bytes(int64_t N, int64_t K);

/* Scratch needed by tw_ternarize_pack: one fp64 row sum per row plus a
 * little header (8*N + 256 bytes, rounded up to 256). */
TW_API size_t tw_ternarize_workspace_bytes(int64_t N, int64_t K);

/*
 * Ternarise W [N x K] fp32 per tensor and pack the codes.
 * Defines: mean = sum|W| / (N*K) accumulated in fp64 in a fixed order (each
 * row summed over k in order, then the row sums over n in order), floored at
 * 1e-5; s = 1/mean; code = clip(rint(W * s), -1, 1) evaluated in fp64 with
 * round-half-to-even.  ("VibeVoice-ASR-BitNet-ONNX" model page, Quantization
 * table: per-tensor s = 1/mean|W|.)
 *   W         [N x K] fp32, read only.
 *   packed    output, packed_bytes >= tw_packed_bytes(N, K); layout above.
 *   mean_abs  output, one double: mean|W| (= 1/s).  May be NULL.
 *   wscale    output, one float: (float)mean, the per-tensor dequant factor
 *             consumed by tw_ternary_linear.  Required.
 *   ws        scratch of ws_bytes >= tw_ternarize_workspace_bytes(N, K).
 * A non-finite W sets TW_ERR_NONFINITE in the device error word (the
 * outputs are then unspecified).
 */
TW_API int tw_ternarize_pack(const float *W, int64_t N, int64_t K, void *packed,
                      size_t packed_bytes, double *mean_abs, float *wscale,
                      void *ws, size_t ws_bytes, tw_stream_t stream);

/*
 * tw_ternarize_pack without scratch arguments, for callers that cannot
 * allocate device memory when they need a matrix packed (for example a
 * plugin inside a host framework that owns the device-memory budget and
 * gives its plugins no allocator, or a loop that must not call cudaMalloc
 * because it may synchronise the device).  The pages have no counterpart of
 * this entry point; it exists only for such callers.
 *
 * Same results as tw_ternarize_pack.  Its scratch (256 + 8*N bytes) lives
 * in a fixed device array inside the library, sized for N <= TW_NOALLOC_MAX_N
 * rows; every GPU that loads the library keeps that array (262,400 bytes)
 * until the process exits.  Larger N returns TW_ERR_SHAPE.  The first call
 * on a device looks the array's device address up (cudaGetSymbolAddress);
 * make that first call before any stream capture.  All calls on a device
 * share the one array, so calls that may run at the same time on the GPU
 * (different streams, no ordering between them) race and corrupt each
 * other's results; order them on one stream.  Allocates no memory.
 */
#define TW_NOALLOC_MAX_N 32768
TW_API int tw_ternarize_pack_noalloc(const float *W, int64_t N, int64_t K,
                                     void *packed, size_t packed_bytes,
                                     double *mean_abs, float *wscale,
                                     tw_stream_t stream);

/*
 * Debug / parity: unpack codes to int8 {-1, 0, 1} row-major [N x K].
 * invalid_count (device, one int32, may be NULL) receives the number of
 * 2-bit fields holding the invalid pattern 3 (those codes are written as 0).
 */
TW_API int tw_unpack_codes(const void *packed, int64_t N, int64_t K, int8_t *codes,
                    int32_t *invalid_count, tw_stream_t stream);

/*
 * Per-token int8 activation quantisation of x [M x K] fp32 by absmax.
 *   amax[m]  = max_k |x[m,k]|                     (fp32, exact)
 *   scale    = 127.0f / amax[m]                   (IEEE fp32 division)
 *   xq[m,k]  = clamp(rint(x[m,k] * scale), -128, 127)   (fp32 multiply,
 *              round-half-to-even); a row with amax == 0 gives xq == 0.
 *   qsum[m]  = sum_k xq[m,k]  (optional, may be NULL; the prefill entry
 *              points use it to fold the +1 code offset back out).
 * The pages name only "fused INT8" operations (xujun.org article,
 * heterogeneous-quantisation section); this is the plainest absmax reading.
 * Non-finite x gives unspecified results.
 */
TW_API int tw_quantize_act(const float *x, int64_t M, int64_t K, int8_t *xq,
                    float *amax, int32_t *qsum, tw_stream_t stream);

/* Scratch needed by tw_ternary_linear for this shape: the int8 rows plus
 * per-token scales (M <= 32: round128(M*K) + 256 bytes; larger M:
 * M*K + 8*M bytes rounded up).  tw_ternary_linear_q needs none. */
TW_API size_t tw_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * y = rescale(quantize(x) * codes^T): the whole layer on one matrix.
 *   acc[m,n] = sum_k code[n,k] * xq[m,k]          (exact int32)
 *   y[m,n]   = ((float)acc * (amax[m] / 127.0f)) * wscale   (fp32)
 * x [M x K] fp32; packed/wscale from tw_ternarize_pack; y [M x N] fp32
 * output; acc_out [M x N] int32 output or NULL.  M <= 32 runs the fused
 * act-quant + decode kernel; larger M quantises into ws and runs the
 * tensor-core prefill kernel.
 */
TW_API int tw_ternary_linear(const float *x, int64_t M, int64_t N, int64_t K,
                      const void *packed, const float *wscale, float *y,
                      int32_t *acc_out, void *ws, size_t ws_bytes,
                      tw_stream_t stream);

/*
 * Same product on activations already quantised by tw_quantize_act:
 * xq [M x K] int8, amax [M] fp32, qsum [M] int32 (required).  ws and
 * ws_bytes are not used (NULL and 0 are fine); they keep the argument list
 * of tw_ternary_linear.
 */
TW_API int tw_ternary_linear_q(const int8_t *xq, const float *amax,
                        const int32_t *qsum, int64_t M, int64_t N, int64_t K,
                        const void *packed, const float *wscale, float *y,
                        int32_t *acc_out, void *ws, size_t ws_bytes,
                        tw_stream_t stream);

/*
 * One projection of a decoder sweep.  All pointers are device pointers.
 * Decode sweeps (M <= 32) read x.  Sweeps of more than 32 tokens read xq,
 * amax and qsum: either as given (from tw_quantize_act; x NULL) or, when x
 * is given too, as written by the sweep itself, which then quantises every
 * such x into its xq, amax and qsum (R2-R4, the same bits as
 * tw_quantize_act) in one launch over all projections before the GEMM.
 */
typedef struct tw_proj_desc {
    const float *x;        /* [M x K] fp32 activations (decode; prefill:   */
                           /* optional, quantised into xq/amax/qsum)       */
    const int8_t *xq;      /* [M x K] int8 activations (prefill)           */
    const float *amax;     /* [M] absmax that goes with xq (prefill)       */
    const int32_t *qsum;   /* [M] row sums of xq (prefill)                 */
    const void *packed;    /* packed codes of W [N x K]                    */
    const float *wscale;   /* one float, mean|W|                           */
    float *y;              /* [M x N] fp32 output                          */
    int32_t *acc_out;      /* [M x N] int32 output, or NULL                */
    int64_t N, K;
} tw_proj_desc;

/* Bytes of the encoded sweep table for `count` projections. */
TW_API size_t tw_sweep_table_bytes(int count);

/*
 * HOST-ONLY.  Validate `count` descriptors (host array) for a sweep over M
 * tokens and encode them into `table` (host memory, table_bytes >=
 * tw_sweep_table_bytes(count)).  The caller copies the table to device
 * memory (64-byte aligned) and passes that copy to
 * tw_decoder_projection_sweep; the table stays valid for as long as the
 * buffers it names do.  Layout: a 64-byte header, one 384-byte record per
 * projection, then one 16-byte entry per projection giving the order in
 * which the tensor-core kernels hand out their units (projections of larger
 * K first).  The records embed TMA descriptors --
 * of each xq (M > 32) and of the packed codes (every M) -- and therefore
 * need the CUDA driver: a decode table encoded where the driver is missing
 * still answers the size queries, but the sweep refuses it (TW_ERR_CUDA).
 */
TW_API int tw_sweep_table_encode(const tw_proj_desc *descs, int count, int64_t M,
                          void *table, size_t table_bytes);

/* The GEMM that a sweep of more than 32 tokens runs. */
#define TW_SWEEP_GEMM_AUTO 0     /* by M: weights expanded into tensor memory */
                                 /* for 33..192 tokens, into shared memory    */
                                 /* above (the measured crossover)            */
#define TW_SWEEP_GEMM_EXPANDED 1 /* weights expanded into shared memory for   */
                                 /* every M > 32                              */

/*
 * HOST-ONLY.  tw_sweep_table_encode with the GEMM of a sweep of more than
 * 32 tokens chosen by the caller: TW_SWEEP_GEMM_AUTO (what
 * tw_sweep_table_encode does) or TW_SWEEP_GEMM_EXPANDED, which runs the
 * expanded-weights GEMM at 33..192 tokens too (to time the two kernels
 * against each other on the caller's own shapes).  Both give the same bits:
 * the int32 sums are exact and the rescale is the same expression.  For
 * M <= 32 the choice is ignored.  Any other value: TW_ERR_SHAPE.
 */
TW_API int tw_sweep_table_encode_gemm(const tw_proj_desc *descs, int count, int64_t M,
                               int gemm, void *table, size_t table_bytes);

/* Scratch needed by tw_decoder_projection_sweep for an encoded HOST table.
 * For decode (M <= 32) it holds 256 bytes of work counters, then the
 * quantised rows of every projection (room for 8, 16 or 32 token rows of K
 * bytes) and their scales; for more tokens (whose callers pass the
 * quantised rows in the descriptors) only the 256 bytes of work counters.
 * It must be zero-filled before its first use with a table; every call
 * leaves the counters zero again (after TW_ERR_TIMEOUT, zero it again). */
TW_API size_t tw_sweep_workspace_bytes(const void *table_host);

/*
 * Run the layer over every projection of an encoded table.  Decode
 * (M <= 32): one quantisation launch, then for M <= 8 one persistent
 * launch of the register (mma.sync) kernel -- more only when M*K of the
 * widest projection does not fit shared memory and the tokens are split
 * into groups -- and for 8 < M <= 32 one launch of the tensor-core decode
 * kernel.  33..192 tokens: one persistent tensor-core launch with the
 * weights in tensor memory (units of 128 weight rows x 64, 96, 128 or 192
 * tokens, the narrowest that holds M, claimed from the counters in the
 * workspace); more tokens (or TW_SWEEP_GEMM_EXPANDED): one persistent
 * tensor-core launch with the weights expanded in shared memory (output
 * tiles of 128 tokens x 256 weight rows dealt out round robin).  Either is
 * preceded by one quantisation launch when some descriptor gives x.
 *   table_host  the host table written by tw_sweep_table_encode (read for the
 *               launch configuration: count, M, sizes);
 *   table_dev   the caller's device copy of the same bytes (64-byte aligned),
 *               which the kernels read.
 * The 196 projections of the synthetic decoder sweep share no data: each
 * has its own x and y.
 */
TW_API int tw_decoder_projection_sweep(const void *table_host, const void *table_dev,
                                void *ws, size_t ws_bytes, tw_stream_t stream);

/* HOST-ONLY.  Number of kernel launches one tw_decoder_projection_sweep call
 * on this encoded table makes (0 for a malformed table). */
TW_API int tw_sweep_launches(const void *table_host);

/*
 * Decoder-layer chain
 * -------------------
 * The projections of consecutive decoder layers with their data
 * dependencies.  Per layer: q, k and v read one input h; attention is the
 * identity over positions (every token attends only to itself, so its
 * output is its own v, each KV head repeated for the query heads of its
 * group); o reads that; h1 = h + o; gate and up read h1; act = SiLU(gate) *
 * up with SiLU(z) = z / (1 + e^-z); down reads act; the layer's output
 * h1 + down replaces h.  This is the decoder layer of the Qwen2.5-1.5B LM
 * ("VibeVoice-ASR-BitNet-ONNX" model page, "Layout": decoder_model_merged
 * maps inputs_embeds and the KV cache to logits) without the parts that need
 * trained weights or a cache: attention scores, the KV cache and the
 * normalisation gains.  Residual adds are single-precision; SiLU uses expf.
 * Decode only: 1 <= M <= 32.
 */
typedef struct tw_chain_buffers {
    float *h;     /* [M x hidden] input of the first layer; output of the last   */
    float *v;     /* [M x kv_dim] output of v                                     */
    float *a;     /* [M x hidden] attention output, the input of o                */
    float *o;     /* [M x hidden] output of o                                     */
    float *h1;    /* [M x hidden] h + o, the input of gate and up                 */
    float *g;     /* [M x inter]  output of gate                                  */
    float *u;     /* [M x inter]  output of up                                    */
    float *act;   /* [M x inter]  SiLU(g) * u, the input of down                  */
    float *d;     /* [M x hidden] output of down                                  */
    int64_t M, hidden, kv_dim, head_dim, inter;
} tw_chain_buffers;

/*
 * One layer as four encoded sweep tables (host bytes and device copies, as
 * for tw_decoder_projection_sweep), encoded for M tokens and the buffers:
 *   qkv   q [hidden x hidden], k and v [kv_dim x hidden]; every x = h;
 *         v's y = v (q's and k's outputs go wherever their descriptors say)
 *   o     [hidden x hidden], x = a, y = o
 *   gu    gate and up [inter x hidden], x = h1, y = g and u
 *   down  [hidden x inter], x = act, y = d
 * acc_out of any descriptor may be set (tests read the integer results).
 */
typedef struct tw_chain_layer {
    const void *qkv_host, *qkv_dev;
    const void *o_host, *o_dev;
    const void *gu_host, *gu_dev;
    const void *down_host, *down_dev;
} tw_chain_layer;

/* HOST-ONLY.  Scratch of tw_decoder_chain: the largest
 * tw_sweep_workspace_bytes of the tables (the sweeps run one after another
 * on one stream and share it; the same zero-fill rule applies).  0 if a
 * table is missing or malformed. */
TW_API size_t tw_chain_workspace_bytes(const tw_chain_layer *layers, int n_layers);

/*
 * Run n_layers layers (host array `layers`, host struct `buf`) in order on
 * `stream`: per layer four sweeps and four element-wise launches (the
 * attention stand-in, the two residual adds and SiLU * up).  Every
 * table is checked on the host against `buf` first -- projection count, N
 * and K, M, and the x and y pointers named above -- and nothing is launched
 * if one does not match (TW_ERR_SHAPE, TW_ERR_NULL, TW_ERR_ALIGN,
 * TW_ERR_CORRUPT or TW_ERR_BUFSIZE).  A launch that fails part-way returns
 * TW_ERR_CUDA with the earlier steps already enqueued; the buffers then hold
 * a partial result.  The caller keeps the tables, buffers, weights and `ws`
 * allocated until the stream has finished the call.
 */
TW_API int tw_decoder_chain(const tw_chain_layer *layers, int n_layers,
                            const tw_chain_buffers *buf, void *ws, size_t ws_bytes,
                            tw_stream_t stream);

/* HOST-ONLY.  Kernel launches of one tw_decoder_chain call (0 if a table is
 * missing or malformed). */
TW_API int tw_chain_launches(const tw_chain_layer *layers, int n_layers);

/*
 * The same chain fused into one persistent kernel per group of up to 8
 * tokens: all layers' stages run in one launch with grid-wide barriers
 * between the dependent stages, and the steps between the projections (the
 * activation quantisation, the rescale, the attention stand-in, the
 * residual adds and SiLU * up) are done inside it.  Each stage's work is
 * split over every SM along rows and k (partial sums are added with integer
 * atomics, exact in any order); the code stream of later stages is fetched
 * while the grid waits at a barrier.  Results are byte-identical to
 * tw_decoder_chain (the same fp32 operations in the same order).
 *
 * tw_chain_plan_encode (HOST-ONLY) checks the layers' tables against `buf`
 * exactly as tw_decoder_chain does and writes a plan of
 * tw_chain_plan_bytes(n_layers) bytes into host memory, for the SM count of
 * the current device; the caller copies it to device memory (64-byte
 * aligned) and keeps both, the tables' buffers and `buf` alive while it is
 * used.  head_dim must be a multiple of 4.
 */
TW_API size_t tw_chain_plan_bytes(int n_layers);
TW_API int tw_chain_plan_encode(const tw_chain_layer *layers, int n_layers,
                                const tw_chain_buffers *buf, void *plan, size_t plan_bytes);

/* HOST-ONLY.  Scratch of tw_decoder_chain_fused for a host plan: 256 bytes
 * of barrier counters, then four int32 sum buffers of 8 rows of the widest
 * stage's outputs.  It must be zero-filled before its first use; every call
 * leaves the counters zero again (after TW_ERR_TIMEOUT, zero it again). */
TW_API size_t tw_chain_fused_workspace_bytes(const void *plan_host);

/* HOST-ONLY.  Kernel launches of one tw_decoder_chain_fused call:
 * ceil(M / 8). */
TW_API int tw_chain_fused_launches(const void *plan_host);

/*
 * Run every layer of an encoded plan (host and device copies) on `stream`:
 * ceil(M / 8) cooperative launches of one CTA per SM, each running all the
 * layers for its tokens.  TW_ERR_UNSUPPORTED if the device has fewer SMs
 * than the plan was encoded for.  Every barrier and copy wait is bounded:
 * a wait that expires is reported by tw_check as TW_ERR_TIMEOUT.
 */
TW_API int tw_decoder_chain_fused(const void *plan_host, const void *plan_dev, void *ws,
                                  size_t ws_bytes, tw_stream_t stream);

/*
 * I8_S linear layer with fused bias and ReLU
 * ------------------------------------------
 * The int8 side of the model: the audio encoder keeps int8 weights and int8
 * activations and replaces GELU by ReLU ("VibeVoice-ASR-BitNet-ONNX" model
 * page, "Quantization" table, row "VAE encoders": I8_S), and its fused int8
 * routines join matmul, bias and ReLU in one pass (aitrends summary,
 * technical features).  The weights carry one absmax scale per tensor (the
 * "_S" format, like the ternary one):
 *   amax_w = max|W|,  wq = clamp(rint(W * (127.0f / amax_w)), -128, 127)
 * (fp32 multiply, IEEE division, half to even; W == 0 gives wq == 0).
 * Activations are quantised per token exactly as tw_quantize_act does.
 *   acc[m, n] = sum_k xq[m, k] * wq[n, k]            (exact int32)
 *   y[m, n]   = ((float)acc * (amax_x[m] / 127.0f)) * (amax_w / 127.0f) + bias[n]
 *               then max(0, y) when relu != 0        (fp32, rounded per step)
 * K must be a positive multiple of 16 (the operands are read as 16-byte
 * rows; k past K reads as zero), N and M any size >= 1.  All pointers are
 * device pointers, 16-byte aligned.
 */

/* HOST-ONLY.  Scratch of tw_i8_linear: the int8 rows and scales of x. */
TW_API size_t tw_i8_workspace_bytes(int64_t M, int64_t K);

/*
 * Quantise the weights of one I8_S layer: W [N x K] fp32 -> wq [N x K] int8
 * (row-major) and amax_w (one float).  A non-finite W sets TW_ERR_NONFINITE
 * in the device error word (tw_check); wq is then unspecified.
 */
TW_API int tw_i8_quantize_weights(const float *W, int64_t N, int64_t K, int8_t *wq,
                                  float *amax_w, tw_stream_t stream);

/*
 * y [M x N] fp32 from int8 activations xq [M x K] with their per-token
 * amax_x [M] (as tw_quantize_act writes them), wq [N x K] and amax_w from
 * tw_i8_quantize_weights, bias [N] fp32 (NULL: no bias), relu 0 or 1.
 * acc_out [M x N] int32 receives the exact accumulators (NULL: not written).
 * One launch on the tensor cores.
 */
TW_API int tw_i8_linear_q(const int8_t *xq, const float *amax_x, int64_t M, int64_t N, int64_t K,
                          const int8_t *wq, const float *amax_w, const float *bias, int relu,
                          float *y, int32_t *acc_out, tw_stream_t stream);

/*
 * The same layer from fp32 activations x [M x K]: quantises x into ws
 * (ws_bytes >= tw_i8_workspace_bytes(M, K)), then runs tw_i8_linear_q.
 */
TW_API int tw_i8_linear(const float *x, int64_t M, int64_t N, int64_t K, const int8_t *wq,
                        const float *amax_w, const float *bias, int relu, float *y,
                        int32_t *acc_out, void *ws, size_t ws_bytes, tw_stream_t stream);

/*
 * Tensor-parallel split of the projections
 * ----------------------------------------
 * Pieces of a Megatron-style split across ranks (one GPU each).  The pages
 * describe single-process inference; the split is this library's own and
 * its result is, by construction, the single-device result bit for bit.
 *  - column-parallel (q, k, v, gate, up): a rank holds rows [n0, n0 + rows)
 *    of W (tw_pack_slice of the whole matrix's codes, with the whole
 *    matrix's wscale) and the whole input; its output is its slice of y.
 *  - row-parallel (o, down): a rank holds input columns [k0, k0 + cols) and
 *    the matching columns of W (tw_pack_slice).  Per token: tw_row_absmax of
 *    its slice, a max all-reduce of those M floats over the ranks,
 *    tw_quantize_act_given with that maximum, tw_ternary_linear_q into its
 *    int32 acc_out, an int32 sum all-reduce of the M x N partial sums, and
 *    tw_rescale_acc.  The collectives are the caller's (NCCL).
 */

/*
 * Copy the codes of the sub-matrix rows [n0, n0 + rows) x columns
 * [k0, k0 + cols) of a packed [N x K] matrix into `out` in the packed layout
 * of a [rows x cols] matrix (out_bytes >= tw_packed_bytes(rows, cols)).
 * n0 a multiple of 16, k0 and cols multiples of 128; rows past the slice in
 * its last 16-row block are written as code 0.  Exact (a byte gather).
 */
TW_API int tw_pack_slice(const void *packed, int64_t N, int64_t K, int64_t n0, int64_t rows,
                         int64_t k0, int64_t cols, void *out, size_t out_bytes,
                         tw_stream_t stream);

/* amax[m] = max_k |x[m, k]| of x [M x K] fp32 (K a multiple of 4); exact. */
TW_API int tw_row_absmax(const float *x, int64_t M, int64_t K, float *amax, tw_stream_t stream);

/*
 * Per-token int8 quantisation with a given per-token absmax (as
 * tw_quantize_act, but amax[m] is an input, e.g. the maximum over the
 * ranks' slices of the row): xq = clamp(rint(x * (127.0f / amax[m])),
 * -128, 127); amax[m] == 0 gives xq == 0; qsum[m] = sum_k xq[m, k] (may be
 * NULL).  K a multiple of 4.
 */
TW_API int tw_quantize_act_given(const float *x, int64_t M, int64_t K, const float *amax,
                                 int8_t *xq, int32_t *qsum, tw_stream_t stream);

/*
 * y [M x N] = ((float)acc * (amax[m] / 127.0f)) * wscale[0]: the rescale
 * every projection epilogue of this library applies, for accumulators
 * summed outside (acc [M x N] int32, amax [M], wscale one float).
 */
TW_API int tw_rescale_acc(const int32_t *acc, int64_t M, int64_t N, const float *amax,
                          const float *wscale, float *y, tw_stream_t stream);

/* Wait for `stream`, then return and clear the device error word of the
 * current device (TW_OK if no kernel reported an error). */
TW_API int tw_check(tw_stream_t stream);

/* Message of the last failing call on this host thread ("" if none). */
TW_API const char *tw_last_error(void);

/*
 * Self-test of the bounded-wait machinery: launch one block that waits on a
 * barrier nothing ever completes, giving up after timeout_ns; the kernel
 * then records TW_ERR_TIMEOUT, which tw_check() returns.  Faults nothing.
 */
TW_API int tw_debug_wait_timeout(uint64_t timeout_ns, tw_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TERNARY_DECODER_H */
