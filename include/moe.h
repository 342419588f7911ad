/*
 * moe.h -- C ABI of libmoe.so: the forward pass of a top-k routed
 * mixture-of-experts SwiGLU FFN layer on NVIDIA B200 (sm_100a).
 *
 * What the layer computes (Zero to Frontier, ch. 13 section 13.1 "Why MoE",
 * "The MoE layer"; kevinluzbetak "Mixture-Of-Experts", routing paragraph):
 *
 *   r   = x W_r (+ b)                    router logits, one per expert, fp32
 *   p   = softmax(r)                     over all E experts
 *   K   = TopK(r, k)                     ties go to the lower expert index
 *   g_i = e^{r_i} / sum_{j in K} e^{r_j} (the same as p_K / sum p_K)
 *   y   = sum_{i in K, kept} g_i FFN_i(x) + FFN_shared(x)
 *   FFN(x) = (SiLU(x W_g) * (x W_u)) W_d
 *   aux = E * sum_i f_i P_i              f_i = routed assignments / (T k),
 *                                        P_i = mean_t p_ti
 *
 * Capacity (AI Engineering Illustrated "Mixture of Experts", "The safety valve
 * is a capacity limit"; jacopoparretti "Mixture of experts, token by token",
 * "A hard limit"; kevinluzbetak capacity example): when capacity_factor > 0,
 * each expert keeps at most C = floor(capacity_factor * T * k / E)
 * assignments, the first C in token order; a dropped assignment contributes
 * 0 (the token keeps its other experts' terms, gates are not renormalised).
 * The shared expert is never dropped and has weight 1.
 *
 * The Switch balance statistic (kevinluzbetak balancing list; jacopoparretti
 * "A penalty") is returned raw, without the trainer's alpha weight.
 *
 * Conventions for every entry point:
 *   - Every pointer is owned by the caller. Device pointers are CUDA device
 *     memory of the current device; host pointers are ordinary (ideally
 *     pinned) host memory. The library allocates no memory.
 *   - Arrays are row-major and dense. Device pointers must be 16-byte aligned.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and return MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE.
 *   - moe_forward is asynchronous on dims->stream; a CUDA launch failure
 *     returns MOE_ERR_CUDA. Bounded device-side waits record a timeout in two
 *     places: the call's own status word inside its workspace (see
 *     moe_workspace_layout_t.status; moe_forward_host_io reports it), and one
 *     device-wide word that moe_get_device_status reads and clears. The
 *     device-wide word is shared by every call on the device: with concurrent
 *     calls (several streams or threads) it cannot tell which call timed out,
 *     and one caller's read clears it for all. Use the per-call word there.
 *   - Calls on one stream are ordered; two calls that share one workspace
 *     must not overlap on the device.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, NaN factor */
  MOE_ERR_UNSUPPORTED = 2,    /* valid layer this library does not run (see limits below) */
  MOE_ERR_WORKSPACE = 3,      /* workspace null, too small or misaligned */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5, /* a device-side bounded wait gave up (moe_get_device_status) */
  MOE_ERR_SCRATCH_LIMIT = 6,  /* moe_forward_no_alloc: the layer needs more scratch than
                                 MOE_NO_ALLOC_WORKSPACE_BYTES */
  MOE_ERR_DEVICE_BOUNDS = 7   /* builds with MOE_DEBUG only: a device-side bounds check on a
                                 permuted row, a segment start or a TMA row coordinate failed
                                 (the access was skipped; outputs undefined) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Number of steps moe_forward enqueues, in order: router logits, routing
 * (softmax / top-k / gates / ranks), scan (counts, capacity, offsets, aux),
 * scatter (permute x rows), gate/up grouped GEMM + SwiGLU, down grouped GEMM
 * + gate scaling, combine (un-permute + shared expert). Each step is one
 * kernel, except the router step with bf16 x (two: the exact bf16 split of W_r
 * and the tensor-core logits) and, with MOE_WEIGHTS_FP8_W8A8, the scatter and
 * down steps (each one more: the x and H quantisers). */
#define MOE_NUM_KERNELS 7

/* Limits of this library: 1 <= k <= 32, k <= E <= 1024; bf16 needs d, d_e, d_s
 * multiples of 64; fp32 needs them multiples of 32; T < 2^31 / max(k, 1);
 * n_group <= 32 and a divisor of E, k <= topk_group * E / n_group; the
 * quantised weight formats need bf16 x and no shared expert (d_s = 0), and
 * MXFP4 needs d and d_e multiples of 256. */

/*
 * Routing variants (gate_mode, selection_bias, n_group / topk_group).
 *   MOE_GATE_RENORM  g = softmax over the chosen logits (the definition above).
 *   MOE_GATE_RAW     g_i = p_i, the softmax over all experts, not renormalised:
 *                    Switch's top-1 form (jacopoparretti "Mixture of experts,
 *                    token by token", "Experts and a router"; kevinluzbetak
 *                    routing example, "some implementations skip the
 *                    renormalisation").
 *   MOE_GATE_SIGMOID affinities s_i = sigmoid(r_i), top-k on s, g = s_K / sum s_K
 *                    (DeepSeek-V3: AI Engineering Illustrated "Mixture of
 *                    Experts", "The router is small but it decides everything").
 *                    Here P_i of the balance statistic is the mean of
 *                    s_i / sum_j s_j over all experts.
 * selection_bias: added to the logit (RENORM, RAW) or to the affinity
 * (SIGMOID) only when choosing the experts; the gates ignore it (DeepSeek-V3's
 * balancing bias: AI Engineering Illustrated, "Fix 2 nudges a bias instead";
 * jacopoparretti, "A bias").
 * Group-limited selection (jacopoparretti, "Smaller experts, more of them": 4 of
 * 8 groups): a group's score is its largest selection score; a token keeps the
 * topk_group best groups (ties to the lower group) and picks its k experts
 * among them.
 */
#define MOE_GATE_RENORM 0
#define MOE_GATE_RAW 1
#define MOE_GATE_SIGMOID 2

/*
 * FP8 expert weights (weight-only quantisation). At small batch, an MoE layer
 * is limited by reading expert weights, and quantising them attacks that
 * directly (AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
 * weigh"; jacopoparretti "Mixture of experts, token by token", "Memory":
 * DeepSeek-V3 ships FP8 weights). Format: E4M3 (bias 7, largest finite 448,
 * round-to-nearest-even, saturating); one fp32 scale per output row,
 * scale = absmax(row) / 448 (1 for an all-zero row), code = E4M3(w / scale).
 * The layer computes with code * scale: the GEMMs stream the codes and decode
 * them on chip to fp16 (exact), and run fp16 x fp16 -> fp32 on the tensor
 * cores, so the routed activations and H are held in fp16 on this path
 * (exact for bf16 inputs with 2^-14 <= |x| <= 65504; larger magnitudes
 * saturate at 65504). x and y stay bf16.
 */
#define MOE_WEIGHTS_DTYPE 0
#define MOE_WEIGHTS_FP8 1
/*
 * FP8 on both GEMM operands (W8A8): the weights as for MOE_WEIGHTS_FP8, and
 * the routed experts' inputs quantised the same way, one fp32 scale per row:
 * each token row of x (absmax over d) and each routed hidden row H (absmax
 * over d_e, from H's fp32 value) becomes E4M3 codes * scale. The expert
 * GEMMs then run E4M3 x E4M3 -> fp32 on the tensor cores, and both scales
 * multiply the accumulator. This
 * changes the numbers (activations carry 3 mantissa bits): it is a different
 * layer from MOE_WEIGHTS_FP8, not a faster route to the same one.
 */
#define MOE_WEIGHTS_FP8_W8A8 2
/*
 * MXFP4 expert weights (weight-only; the 4-bit format gpt-oss quantises its
 * experts to: AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
 * weigh"). The pages give no format details; this library follows the Open
 * Compute microscaling convention. Each block of 32 consecutive weights of a
 * row (along K) shares X = floor(log2(absmax of the block)) - 2 (X = 0 for an
 * all-zero block); each weight becomes the E2M1 value (magnitudes 0, 0.5, 1,
 * 1.5, 2, 3, 4, 6) nearest to w / 2^X, ties to the even mantissa, saturating
 * at +-6; the layer computes with code * 2^X. Storage, per weight stack:
 *   codes        uint8 [rows, K / 2]: two codes per byte, the even-K element in
 *                the low nibble (bit 3 = sign, bits 2..1 = exponent, bit 0 =
 *                mantissa); passed as W_g, W_u, W_d;
 *   block scales uint8 [rows, K / 32]: X + 127 (E8M0); the three stacks' one
 *                after another form moe_dims.weight_block_scales;
 *   row factors  fp32 [rows]: 2^(the largest X among the row's non-zero blocks),
 *                1 for an all-zero row; the three stacks' one after another form
 *                moe_dims.weight_scales.
 * moe_quantize_mxfp4 writes all three. The GEMMs stream the codes, decode them
 * on chip to fp16 (the E2M1 value times 2^(X - X_row), exact while
 * X >= X_row - 23; weights of smaller blocks are rounded to multiples of
 * 2^(X_row - 24)) and apply the row factor to the fp32 accumulator. As with
 * FP8 weight-only, the routed activations and H are held in fp16 on this path.
 * Needs bf16 x, no shared expert, and d, d_e multiples of 256.
 */
#define MOE_WEIGHTS_MXFP4 3

typedef struct {
  int64_t T;                 /* tokens in this call (0 allowed: empty batch) */
  int32_t d;                 /* model width */
  int32_t d_e;               /* routed expert hidden width */
  int32_t d_s;               /* shared expert hidden width; 0 = no shared expert */
  int32_t dtype;             /* moe_dtype of x, W_g, W_u, W_d, W_shared and y */
  int32_t gate_mode;         /* MOE_GATE_RENORM (0), MOE_GATE_RAW (1) or MOE_GATE_SIGMOID (2),
                                see "Routing variants" above */
  const float* router_bias;  /* device [E] fp32 added to the logits before softmax
                                and top-k, or NULL */
  void* workspace;           /* device scratch of >= moe_workspace_size() bytes,
                                256-byte aligned, owned by the caller */
  size_t workspace_bytes;
  void* stream;              /* cudaStream_t to enqueue on; NULL = default stream */
  void* const* events;       /* optional cudaEvent_t[2*MOE_NUM_KERNELS]; when non-NULL,
                                events[2i] / events[2i+1] are recorded on `stream`
                                right before / after step i (NULL entries skipped);
                                with MOE_WEIGHTS_FP8_W8A8 the x quantiser falls in the
                                scatter step and the H quantiser in the down step */
  const float* selection_bias; /* device [E] fp32 added to the selection scores only
                                  (who is picked, not the gates), or NULL */
  int32_t n_group;           /* group-limited selection: experts form n_group contiguous
                                groups of E / n_group; 0 or 1 = no groups */
  int32_t topk_group;        /* groups a token may pick from (1 <= topk_group <= n_group) */
  int32_t weight_format;     /* MOE_WEIGHTS_DTYPE (0): W_g, W_u, W_d in `dtype`;
                                MOE_WEIGHTS_FP8 (1): E4M3 codes (uint8) with per-row scales,
                                see moe_quantize_fp8 (bf16 activations, no shared expert);
                                MOE_WEIGHTS_FP8_W8A8 (2): the same weights, and E4M3
                                activations inside the experts (see above);
                                MOE_WEIGHTS_MXFP4 (3): packed E2M1 codes with block scales
                                and row factors, see above and moe_quantize_mxfp4 */
  const float* weight_scales; /* MOE_WEIGHTS_FP8(_W8A8): device fp32, the per-row scales of the
                                 three stacks one after another: W_g [E*d_e], W_u [E*d_e],
                                 W_d [E*d] (what moe_quantize_fp8 writes for each stack);
                                 MOE_WEIGHTS_MXFP4: the row factors, in the same order */
  uint64_t wait_timeout_ns;  /* limit of each device-side mbarrier wait in the GEMM
                                kernels; 0 = default (4 s). A tiny value makes the waits
                                expire on purpose: the kernels then record
                                MOE_ERR_DEVICE_TIMEOUT, let their in-flight copies and
                                MMAs land, free TMEM and return (outputs undefined), and
                                the context stays usable. */
  const uint8_t* weight_block_scales; /* MOE_WEIGHTS_MXFP4 only: device uint8 E8M0 block
                                 scales, 16-byte aligned, of the three stacks one after
                                 another: W_g [E*d_e*(d/32)], W_u [E*d_e*(d/32)],
                                 W_d [E*d*(d_e/32)] (what moe_quantize_mxfp4 writes);
                                 ignored otherwise */
} moe_dims;

/* Bytes of device workspace moe_forward needs for this layer (0 on invalid
 * arguments). Depends on T, d, d_e, d_s, dtype, E, k and capacity_factor. */
MOE_API size_t moe_workspace_size(const moe_dims* dims, int E, int k, float capacity_factor);

/* Capacity C = floor(capacity_factor * T * k / E) the forward pass applies,
 * or -1 when capacity_factor <= 0 (no limit). */
MOE_API int64_t moe_capacity(int64_t T, int E, int k, float capacity_factor);

/*
 * Forward pass of the routed MoE FFN layer (see top of file).
 *   x        device [T, d]            dtype
 *   W_r      device [E, d]            fp32 (the router's d x E matrix, stored expert-major)
 *   W_g, W_u device [E, d_e, d]       dtype (nn.Linear weight layout: K contiguous),
 *                                    or uint8 E4M3 codes with MOE_WEIGHTS_FP8(_W8A8)
 *   W_d      device [E, d, d_e]       dtype (or uint8 codes)
 *   W_shared device, packed [gate (d_s x d) | up (d_s x d) | down (d x d_s)], or
 *            NULL when dims->d_s == 0
 *   y        device [T, d]            dtype, written (every row)
 *   aux      device float[1]          written: E * sum_i f_i P_i (0 when T == 0)
 *   counts   device int32[E]          written: routed assignments per expert,
 *                                     before the capacity cut
 * Enqueues MOE_NUM_KERNELS kernels on dims->stream (two more, the x and H
 * quantisers, with MOE_WEIGHTS_FP8_W8A8), no host synchronisation.
 */
MOE_API moe_status moe_forward(const moe_dims* dims,
                       const void* x, const float* W_r, const void* W_g,
                       const void* W_u, const void* W_d, const void* W_shared,
                       int E, int k, float capacity_factor,
                       void* y, float* aux, int32_t* counts);

/*
 * End-to-end variant for callers holding the activations in host memory: the
 * same forward pass, bracketed by the copies. Copies x_host -> x_dev, runs
 * moe_forward, copies y_dev -> y_host, aux_dev -> aux_host and counts_dev ->
 * counts_host, all on dims->stream, then synchronises that stream. If the pass
 * itself was enqueued, it returns MOE_ERR_DEVICE_TIMEOUT when a device-side wait
 * of this call gave up (read from the call's own status word, so concurrent
 * calls on other streams do not see each other's timeouts), else MOE_OK.
 * Weights stay device pointers. x_host / y_host should be pinned for full copy
 * bandwidth.
 */
MOE_API moe_status moe_forward_host_io(const moe_dims* dims,
                               const void* x_host, void* x_dev,
                               const float* W_r, const void* W_g, const void* W_u,
                               const void* W_d, const void* W_shared,
                               int E, int k, float capacity_factor,
                               void* y_dev, void* y_host,
                               float* aux_dev, float* aux_host,
                               int32_t* counts_dev, int32_t* counts_host);

/* Where moe_forward keeps its routing results inside the workspace (byte
 * offsets from dims->workspace), so that callers and tests can read them after
 * the call. Valid until the next call that uses the same workspace. */
typedef struct {
  size_t logits;      /* fp32 [T, E]    router logits x W_r (bias not included) */
  size_t topk_idx;    /* int32 [T, k]   chosen experts, descending logit */
  size_t gates;       /* fp32 [T, k]    gates of those experts */
  size_t slot_pos;    /* int32 [T, k]   row of each assignment in the permuted
                                        buffers, or -1 when dropped */
  size_t probsum;     /* fp64 [E]       sum over tokens of the full softmax */
  size_t tile_start;  /* int32 [E + 1]  first 128-row tile of each expert's
                                        segment; [E] = number of routed tiles */
  size_t xp;          /* dtype [rows_max, d]   x rows grouped by expert */
  size_t h;           /* dtype [rows_max, d_e] SwiGLU hidden rows (fp32 with
                         MOE_WEIGHTS_FP8_W8A8; fp16 with the other quantised formats) */
  size_t yrows;       /* dtype [rows_max, d]   gate-scaled expert outputs */
  int64_t rows_max;   /* rows reserved for the permuted buffers */
  int64_t capacity;   /* C, or -1 */
  /* MOE_WEIGHTS_FP8_W8A8 only (0 otherwise); xp then holds E4M3 codes
   * [rows_max, d] (row stride d bytes) */
  size_t xscale;      /* fp32 [rows_max]       scale of each permuted x row */
  size_t hq;          /* uint8 [rows_max, d_e] E4M3 codes of the hidden rows */
  size_t hscale;      /* fp32 [rows_max]       scale of each hidden row */
  size_t status;      /* int32: this call's status word, 0 when no device-side wait of
                         this call gave up, nonzero otherwise (valid once the call's
                         stream has been synchronised; cleared at the start of each call) */
} moe_workspace_layout_t;

MOE_API moe_status moe_workspace_layout(const moe_dims* dims, int E, int k, float capacity_factor,
                                moe_workspace_layout_t* out);

/* Status of the device-side bounded waits (and, in MOE_DEBUG builds, bounds
 * checks) since the last read, for the current device: reads and clears the
 * device-wide word in one atomic exchange. Call after synchronising the
 * stream(s) used. The word is shared by every call on the device; to attribute
 * a timeout to one of several concurrent calls, read that call's own status
 * word (moe_workspace_layout_t.status) instead. Returns MOE_OK,
 * MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS, or MOE_ERR_CUDA if it cannot
 * be read. */
MOE_API moe_status moe_get_device_status(void);

/* Static, human-readable name of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/*
 * Quantise `rows` rows of `cols` weights (device, `dtype` = MOE_BF16 or MOE_F32,
 * row-major) to E4M3 codes (device uint8 [rows, cols]) and per-row scales
 * (device fp32 [rows]) with the rule above, asynchronously on `stream`. For a
 * routed expert stack, W_g [E, d_e, d] is rows = E * d_e, cols = d (likewise
 * W_u), and W_d [E, d, d_e] is rows = E * d, cols = d_e. Writing the three
 * stacks' scales one after another gives moe_dims.weight_scales. Returns
 * MOE_ERR_INVALID_ARG for null pointers, cols not a multiple of 16, rows < 0,
 * a bad dtype, or w / codes not 16-byte aligned (nothing is launched),
 * MOE_ERR_CUDA on launch failure.
 */
MOE_API moe_status moe_quantize_fp8(const void* w, int32_t dtype, int64_t rows, int32_t cols,
                                    uint8_t* codes, float* scales, void* stream);

/*
 * The weights an FP8 layer computes with: out[r][c] = value(codes[r][c]) *
 * scales[r] (device fp32 [rows, cols]), each code decoded exactly by the
 * routine the GEMM kernels use, the product rounded once to fp32. For
 * checking a quantised stack or materialising it. Codes 0x7F / 0xFF (E4M3
 * NaN, never written by moe_quantize_fp8) are outside the contract. Returns
 * MOE_ERR_INVALID_ARG for null pointers, rows < 0, cols not a multiple of 16,
 * or codes / out not 16-byte aligned (nothing is launched), MOE_ERR_CUDA on
 * launch failure.
 */
MOE_API moe_status moe_dequantize_fp8(const uint8_t* codes, const float* scales, int64_t rows,
                                      int32_t cols, float* out, void* stream);

/*
 * MXFP4 quantisation of `rows` rows of `cols` weights (device, `dtype` =
 * MOE_BF16 or MOE_F32, row-major; cols a multiple of 32) with the rule above,
 * asynchronously on `stream`: codes (device uint8 [rows, cols / 2], 16-byte
 * aligned), block scales (device uint8 [rows, cols / 32]) and row factors
 * (device fp32 [rows]). For a routed expert stack, W_g [E, d_e, d] is
 * rows = E * d_e, cols = d (likewise W_u), and W_d [E, d, d_e] is rows = E * d,
 * cols = d_e. Returns MOE_ERR_INVALID_ARG for null pointers, rows < 0, cols not
 * a multiple of 32, a bad dtype, or w / codes not 16-byte aligned (nothing is
 * launched), MOE_ERR_CUDA on launch failure.
 */
MOE_API moe_status moe_quantize_mxfp4(const void* w, int32_t dtype, int64_t rows, int32_t cols,
                                      uint8_t* codes, uint8_t* block_scales, float* row_factors,
                                      void* stream);

/*
 * The weights an MXFP4 layer computes with: out[r][c] = value(code) * 2^X of
 * its block (device fp32 [rows, cols]), built by the routine the GEMM kernels
 * use (fp16 code * 2^(X - X_row), then times the row factor in fp32), so it is
 * exact under the same condition. For checking a quantised stack or
 * materialising it. Returns MOE_ERR_INVALID_ARG for null pointers, rows < 0,
 * cols not a multiple of 32, or codes / out not 16-byte aligned (nothing is
 * launched), MOE_ERR_CUDA on launch failure.
 */
MOE_API moe_status moe_dequantize_mxfp4(const uint8_t* codes, const uint8_t* block_scales,
                                        const float* row_factors, int64_t rows, int32_t cols,
                                        float* out, void* stream);

/*
 * moe_forward for callers that cannot allocate device memory. The pages have
 * no counterpart: this is a deployment entry point, not part of the method.
 *
 * Who needs it: code that runs inside a host which owns the device memory,
 * e.g. a plugin loaded into an inference server that has reserved all free
 * device memory for its own pool (a cudaMalloc there fails or would steal from
 * the pool), or a plain C caller with no allocator of its own. Such callers
 * cannot provide moe_forward's caller-owned workspace.
 *
 * Instead this call uses one scratch array of MOE_NO_ALLOC_WORKSPACE_BYTES
 * (64 MiB) that lives in the library itself as a statically sized device
 * array: every GPU that loads the library holds it until the process exits.
 * A layer fits when moe_workspace_size() for it is at most
 * MOE_NO_ALLOC_WORKSPACE_BYTES; that is the test to use. The size grows with
 * the permuted rows, T*k plus up to 127 padding rows per expert (each
 * expert's segment is padded to 128 rows), times d and d_e. One example: the
 * Mixtral-shaped layer (d=4096, E=8, d_e=14336, k=2) fits up to T = 128
 * tokens per call (about 58 MB). The call allocates nothing: no cudaMalloc,
 * no cudaFree, no allocating library routine.
 *
 * Arguments and results are exactly those of moe_forward, except that
 * dims->workspace and dims->workspace_bytes are ignored. Inputs and outputs
 * are still caller-owned device memory.
 *
 * Errors: those of moe_forward, plus MOE_ERR_SCRATCH_LIMIT, returned before
 * anything is enqueued, when moe_workspace_size() for this layer exceeds
 * MOE_NO_ALLOC_WORKSPACE_BYTES.
 *
 * Set-up: the first call on each device looks up the device address of the
 * scratch array (cudaGetSymbolAddress) with that device current, and caches
 * it for the life of the process. Make that first call before any stream
 * capture. Resetting the device (cudaDeviceReset, or tearing down and
 * re-creating its primary context) after that first call is not supported:
 * the cached address would be stale.
 *
 * Sharing: every call, on every stream, uses the same scratch array, which
 * keeps the previous call's contents. The pass writes every scratch byte it
 * later reads, so nothing has to start at zero. Calls that overlap on the GPU
 * (for example, concurrent calls on two streams) race on the scratch and
 * produce undefined results. Serialise them, e.g. on one stream.
 */
#define MOE_NO_ALLOC_WORKSPACE_BYTES ((size_t)64 << 20)
MOE_API moe_status moe_forward_no_alloc(const moe_dims* dims,
                                        const void* x, const float* W_r, const void* W_g,
                                        const void* W_u, const void* W_d, const void* W_shared,
                                        int E, int k, float capacity_factor,
                                        void* y, float* aux, int32_t* counts);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
