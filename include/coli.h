/*
 * coli.h -- C ABI of libcoli, a B200 (sm_100a) implementation of one
 * GLM-5.2-shaped MoE layer forward: sigmoid router with correction-bias
 * top-k, token->expert bucketing, SwiGLU experts with packed int4 weights
 * (one F32 scale per row) and Q8_0 int8 activations reduced as integer dot
 * products, and the score-weighted combine plus the shared expert.
 *
 * Sources (page title, then section):
 *  [W] "GLM-5.2-colibri-int4架构解析MoE专家混合与INT4量化原理" (wmrh.cn):
 *      "GLM-5.2的MoE实现", "MoE的工作原理", "GLM-5.2-colibri-int4的量化流程",
 *      "高级配置选项 / 路由策略定制", "量化保留模块".
 *  [C] "Colibri：在笔记本上跑744B参数的AI模型", "关键特性".
 *  [D] "如何在普通电脑上运行 7440 亿参数神经网络" (devtrends.cc),
 *      "引擎是如何工作的".
 *  [H] HN summary (hn.213312.xyz, article 48842459), "已实现的功能".
 *
 * Conventions for every entry point:
 *  - Data pointers are DEVICE pointers (CUDA global memory) owned by the
 *    caller and 16-byte aligned; the library keeps no reference after the
 *    call returns.  `stream` is a cudaStream_t (NULL = the legacy stream).
 *  - Calls are asynchronous and stream-ordered.  A returned COLI_OK means
 *    the work was validated and enqueued; results are ready once the stream
 *    has been synchronised.
 *  - The library allocates no device memory.  Scratch comes from the
 *    caller's `workspace` (size from coli_moe_workspace_bytes).
 *  - Host-detectable errors (null or misaligned pointers, unsupported
 *    shapes, a workspace that is too small) return COLI_EINVAL at once and
 *    enqueue nothing; a failed launch returns COLI_ECUDA.  coli_last_error()
 *    then gives a message (per calling thread).  Device-side problems are
 *    recorded in the workspace's status word and reported by
 *    coli_sync_status.
 *  - n_tok == 0 is a no-op that returns COLI_OK.
 *  - The first call of a forward path on a device sets kernel attributes
 *    (shared-memory opt-ins) and looks up the tensor-map encoder; make one
 *    call of each path (decode: <= 16 tokens, prefill: more) before capturing
 *    calls into a CUDA graph.  Captured calls replay the device pointers and
 *    sizes they were captured with.
 *  - Weights are row-major [out x in]; an int4 row is in/2 bytes, element
 *    2j in the low nibble of byte j, two's complement, plus one F32 scale.
 *  - Results follow the written float-evaluation contracts (router R, row
 *    fold F, combine C) so they can be compared bit for bit with a second
 *    implementation: see the design notes.
 */
#ifndef COLI_H
#define COLI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_EINVAL = 1,   /* bad argument: nothing was enqueued */
    COLI_ENOMEM = 2,   /* workspace too small */
    COLI_ECUDA = 3,    /* a CUDA call or kernel launch failed */
    COLI_ETIMEOUT = 4, /* a bounded device-side wait gave up */
    COLI_EDEVICE = 5   /* a device-side check recorded an error */
} coli_status;

/* Layer shape and routing options ([W] "GLM-5.2的MoE实现": hidden 6144,
 * expert inter 2048, 256 routed experts, 1 shared, 8 per token;
 * [W] "路由策略定制": routed_scaling_factor, norm_topk_prob).
 * weight_bits: 4 (packed int4, also when 0) or 8 (int8 expert weights, the
 * pages' int8 kernel variant, [C] "关键特性"; same per-row F32 scale).
 * Limits: hidden % 128 == 0; inter % 32 == 0; shared_inter % 32 == 0;
 * 1 <= top_k <= min(n_experts, 16); n_experts <= 512; 0 <= n_shared <= 4.
 * int8 weights need inter % 128 == 0 (they run on the streaming kernel of
 * a prepared layer for <= 16 tokens, else on the tensor-core kernels). */
typedef struct {
    int32_t hidden;
    int32_t inter;
    int32_t n_experts;
    int32_t top_k;
    int32_t n_shared;
    int32_t shared_inter;
    int32_t norm_topk_prob;      /* nonzero: renormalise the selected scores */
    float routed_scaling_factor; /* multiplies every routed weight */
    int32_t weight_bits;         /* 4 (or 0) or 8 */
} coli_moe_config;

/* One expert's weights (device pointers): packed int4 rows of in/2 bytes
 * (weight_bits 4) or int8 rows of `in` bytes (weight_bits 8). */
typedef struct {
    const uint8_t* gate_q; /* [inter x hidden*bits/8] */
    const float* gate_s;   /* [inter] */
    const uint8_t* up_q;   /* [inter x hidden*bits/8] */
    const float* up_s;     /* [inter] */
    const uint8_t* down_q; /* [hidden x inter*bits/8] */
    const float* down_s;   /* [hidden] */
} coli_expert;

/* One MoE layer.  `experts` and `shared` are HOST arrays (n_experts and
 * n_shared entries) of device-pointer sets; the router stays F32
 * ([W] "量化保留模块").  `prepared` is the layer's streaming copy
 * (coli_moe_prepare) or NULL: with it, decode batches of up to 16 tokens
 * read the experts from that copy (same results, bit for bit); without it,
 * or for other batch sizes, the kernels read the row-major weights. */
typedef struct {
    coli_moe_config cfg;
    const float* w_router;      /* [n_experts x hidden] F32, device */
    const float* bias;          /* [n_experts] F32 correction bias, device */
    const coli_expert* experts; /* host array [n_experts] */
    const coli_expert* shared;  /* host array [n_shared] */
    const void* prepared;       /* device, 256-byte aligned, or NULL */
} coli_moe_layer;

/* Per-row int4 weight quantiser ([W] "GLM-5.2-colibri-int4的量化流程":
 * rint, one F32 scale per row, packed into U8).  For each row:
 * scale = absmax/7; q = rint(w/scale) clamped to [-8,7] (half to even); an
 * all-zero row gets scale 0.  w: [rows x cols] F32; q_out: [rows x cols/2]
 * bytes; scale_out: [rows] F32.  cols must be a positive multiple of 32. */
coli_status coli_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q_out,
                                    float* scale_out, void* stream);

/* Per-row int8 weight quantiser, the int8 variant of the expert weights
 * ([C] "关键特性": quantisation kernels int8 / packed int4 / packed int2;
 * the int4 recipe of [W] "GLM-5.2-colibri-int4的量化流程" with the int8
 * range): scale = absmax/127; q = rint(w/scale) clamped to [-127,127] (half
 * to even); an all-zero row gets scale 0.  w: [rows x cols] F32; q_out:
 * [rows x cols] int8; scale_out: [rows] F32.  cols a positive multiple of 32. */
coli_status coli_quantize_rows_int8(const float* w, int64_t rows, int64_t cols, int8_t* q_out, float* scale_out,
                                    void* stream);

/* FP8 -> int4 requantiser, the offline converter's step on the GPU
 * ([W] "GLM-5.2-colibri-int4的量化流程": the source model is FP8 e4m3,
 * dequantised to F32, then quantised per row as coli_quantize_rows_int4;
 * its config gives weight_block_size [128, 128]).
 * w8 [rows x cols] e4m3 codes (bit 7 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; 0x7F / 0xFF are NaN); block_factors
 * [ceil(rows/block) x ceil(cols/block)] F32, row-major: element (r, c) is
 * e4m3(w8[r, c]) * block_factors[r / block, c / block] (one F32 multiply;
 * the stored factor multiplies the code's value), and an element whose
 * product is not finite counts as 0.  Outputs as coli_quantize_rows_int4:
 * q_out [rows x cols/2] packed int4, scale_out [rows] F32.
 * cols % 32 == 0; block a positive multiple of 8 (128 for the GLM-5.2 FP8
 * checkpoint).  Integer and F32 results are exact (bit-reproducible). */
coli_status coli_requantize_fp8_int4(const uint8_t* w8, const float* block_factors, int64_t rows, int64_t cols,
                                     int32_t block, uint8_t* q_out, float* scale_out, void* stream);

/* Q8_0-style activation quantiser ([C] "关键特性": Q8_0 风格 int8 激活).
 * Per 32-element block of each token: d = absmax/127 (F32);
 * q = rint(x/d) clamped to [-127,127]; an all-zero block gets d = 0.
 * x: [n_tok x dim] F32; q_out: [n_tok x dim] int8; scale_out: [n_tok x dim/32].
 * dim must be a positive multiple of 32. */
coli_status coli_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q_out,
                                 float* scale_out, void* stream);

/* Router ([W] "MoE的工作原理", "路由策略定制"; [C] DeepSeek-V3 风格的 sigmoid
 * 路由器).  scores[t,e] = sigmoid(x_t . W_r[e]) (F32, contract R); the top_k
 * experts by scores + bias (ties to the lower index) in rank order go to
 * topk_idx [n_tok x top_k]; topk_w [n_tok x top_k] gets the unbiased scores,
 * divided by their sum when norm_topk_prob, times routed_scaling_factor.
 * scores [n_tok x n_experts] is an optional output: pass NULL to keep the
 * scores on chip (one kernel; idx and w are the same bits either way). */
coli_status coli_moe_route(const coli_moe_layer* layer, const float* x, int64_t n_tok, float* scores,
                           int32_t* topk_idx, float* topk_w, void* stream);

/* Bucketing, the pages' "batched MoE" ([H] "已实现的功能"; [D] 合并对相同
 * 专家的请求): counts[e] = number of (token, slot) pairs routed to e;
 * offsets = exclusive prefix sum [n_experts + 1]; perm [n_tok*top_k] lists
 * the flat pair ids t*top_k + k sorted by (expert, token).  Integer output,
 * unique.  Needs n_experts <= 512. */
coli_status coli_moe_bucket(const int32_t* topk_idx, int64_t n_tok, int32_t top_k, int32_t n_experts,
                            int32_t* counts, int32_t* offsets, int32_t* perm, void* stream);

/* One SwiGLU expert on n_tok Q8 tokens ([C] integer dot kernels):
 * g = gate.x, u = up.x (int4 x Q8 block dots, contract F), h = SiLU(g)*u,
 * h re-quantised to Q8_0, y = down.h.  xq [n_tok x hidden] int8,
 * xs [n_tok x hidden/32] F32, y_out [n_tok x hidden] F32.  `expert` points
 * to ONE host-side coli_expert.  Workspace: coli_moe_workspace_bytes(cfg,
 * n_tok) bytes is always enough.  int4 weights only (weight_bits 4).  This
 * is the reference-shape entry point:
 * it runs the general expert kernels (one CTA per 32 outputs), which follow
 * the same contracts and give the same bits as the layer forward's streaming
 * and tensor-core kernels, but it is not the tuned path and carries no
 * performance claim. */
coli_status coli_moe_expert_ffn(const coli_moe_config* cfg, const coli_expert* expert, const int8_t* xq,
                                const float* xs, int64_t n_tok, float* y_out, void* workspace,
                                size_t ws_bytes, void* stream);

/* The layer: out[t] = sum_k w[t,k] * E_{idx[t,k]}(x_t) + sum_s S_s(x_t)
 * ([W] "MoE的工作原理" weighted combine; shared experts always on).
 * x, out: [n_tok x hidden] F32 (may not alias).  Each selected expert's
 * weights are read once for all the tokens routed to it. */
coli_status coli_moe_layer_forward(const coli_moe_layer* layer, const float* x, int64_t n_tok,
                                   float* out, void* workspace, size_t ws_bytes, void* stream);

/* A pre-norm stack of MoE layers: x_{l+1} = x_l + MoE_l(RMSNorm(x_l)), with
 * RMSNorm(x) = x / sqrt(mean(x^2) + eps) (weight 1).  layers: host array of
 * n_layers layers with the same cfg.  x, out: [n_tok x hidden]. */
coli_status coli_moe_stack_forward(const coli_moe_layer* layers, int32_t n_layers, const float* x,
                                   int64_t n_tok, float eps, float* out, void* workspace,
                                   size_t ws_bytes, void* stream);

/* RMSNorm alone (weight 1): y = x * (1/sqrtf(sum(x^2)/dim + eps)), the sum
 * of squares evaluated by contract R (element i feeds accumulator
 * (i/4) mod 32, each an fmaf chain in ascending i from +0, then the 32
 * accumulators added left to right); dim % 128 == 0.  x, y: [n_tok x dim]. */
coli_status coli_rmsnorm(const float* x, int64_t n_tok, int64_t dim, float eps, float* y, void* stream);

/* The layer's streaming copy ([H] "已实现的功能", batched MoE: one read of
 * an expert per layer; [D] "引擎是如何工作的": an expert's matrices are
 * read as one contiguous piece).  The same weight bytes and F32 row scales
 * as the row-major weights, reordered once so that the decode kernel moves
 * each step of a warp's work with one bulk copy: a step ("stage") is 32
 * rows x 256 bytes (8 KB: 16 blocks of packed int4, or 8 blocks of int8
 * stored as their even then odd elements), the 16-byte chunks of a stage row
 * XOR-rotated by the row index.  Gate/up: half units of 16 gate rows and
 * the 16 matching up rows, hidden/32/16 stages each.  Down: units of 32
 * rows, or of 16 rows whose two 256-byte pieces per stage sit in stage rows
 * r and r + 16 when every row spans an even number of whole stages (the
 * GLM-5.2 shape).  Per expert (routed 0..n_experts-1, then shared): gate/up
 * half units, down units, then the scales (gate, up, down), padded to 256
 * bytes; GLM-5.2 shape: 18.9 MB per expert, 4.86 GB per layer, the size of
 * the row-major weights.  coli_moe_prepared_bytes: bytes for the layer (0
 * if cfg is invalid or the shape has no streaming layout: hidden and inter
 * multiples of 128, and each of hidden/32 and inter/32 either a multiple of
 * the blocks of a 256-byte row (16 int4, 8 int8) or a power-of-two number
 * of 16-byte chunks below it).  coli_moe_prepare: writes the copy of
 * `layer`'s weights into `prepared` (device, 256-byte aligned, `bytes` >=
 * coli_moe_prepared_bytes; caller-owned), stream-ordered; the row-major
 * weights are only read.  Re-run it after changing the weights.  Store the
 * pointer in layer->prepared to use it. */
size_t coli_moe_prepared_bytes(const coli_moe_config* cfg);
coli_status coli_moe_prepare(const coli_moe_layer* layer, void* prepared, size_t bytes, void* stream);

/* Bytes of workspace that coli_moe_layer_forward, coli_moe_stack_forward and
 * coli_moe_expert_ffn need for up to max_tokens tokens (0 if cfg is
 * invalid). */
size_t coli_moe_workspace_bytes(const coli_moe_config* cfg, int64_t max_tokens);

/* Message for the last non-OK status returned on the calling thread. */
const char* coli_last_error(void);

/* Test hook (packed int4 weights): the per-32-block int32 partial sums of one expert matrix
 * (which: 0 gate, 1 up, 2 down) against n_tok Q8 vectors, computed by the
 * same device routine as the expert kernels:
 * isum_out[t, r, b] = sum_{j<32} q_w[r, 32b+j] * xq[t, 32b+j],
 * isum_out is [n_tok x rows x dim_in/32] int32. */
coli_status coli_debug_block_partials(const coli_expert* expert, int32_t which, const int8_t* xq,
                                      int64_t n_tok, int64_t dim_in, int64_t rows, int32_t* isum_out,
                                      void* stream);

/* The layer forward for callers that cannot allocate device memory: hosts
 * that own every device allocation and give a plugin no allocator to fill
 * `workspace` from, and serving loops that must not call cudaMalloc after
 * start-up because it can synchronise the device and stall all streams.
 * (This entry point has no counterpart on the pages: the engine they
 * describe runs on CPU memory.)
 * Same arguments and results as coli_moe_layer_forward minus the workspace:
 * the scratch is a fixed 8 MiB array inside the library, which every GPU
 * that loads the library holds until the process exits.  A call whose
 * scratch need (coli_moe_workspace_bytes(&layer->cfg, n_tok)) exceeds 8 MiB
 * is rejected with COLI_EINVAL and a message naming both sizes -- e.g. the
 * GLM-5.2 shape (hidden 6144, inter 2048, 256 experts, top-8, 1 shared)
 * fits up to 22 tokens per call.  n_tok outside [0, 2^24] is rejected with
 * COLI_EINVAL before any size is computed.  The first call on each device
 * looks up the array's device address with that device current and keeps
 * it for the life of the process (a device reset invalidates it: do not call
 * this entry point on a device after cudaDeviceReset); make that first call
 * before any stream capture.  Every call shares the one array,
 * so calls that can overlap on the GPU (different streams, or different
 * host threads on one device) race: order them on one stream.  The array
 * keeps the last call's contents; nothing in it needs to start at zero.
 * Allocates nothing (no cudaMalloc, no cudaFree). */
coli_status coli_moe_layer_forward_noalloc(const coli_moe_layer* layer, const float* x, int64_t n_tok,
                                           float* out, void* stream);

/* Test hook: arms a capture of every per-32-block int32 partial sum that the
 * NEXT coli_moe_layer_forward call on this thread computes, taken inside the
 * expert kernels that run (the streaming kernel of a prepared layer, or the
 * tensor-core kernels: the same kernels with the sums also stored; other
 * calls return COLI_EINVAL and consume the arming).  isum_out (device,
 * 16-byte aligned, n_words int32) receives, for token t and rank k of its
 * routed experts (row t*(K+S) + k) and for shared expert s (row
 * t*(K+S) + K + s), P = 2*inter*(hidden/32) + hidden*(inter/32) words:
 * gate [inter][hidden/32], up [inter][hidden/32], down [hidden][inter/32],
 * where entry [o][b] = sum_{j<32} q_w[o, 32b+j] * q_in[32b+j] (q_in: the
 * token's Q8 x for gate/up, its Q8 h for down).  The forward fails with
 * COLI_EINVAL if n_words < n_tok*(K+S)*P. */
coli_status coli_debug_capture_partials(int32_t* isum_out, size_t n_words);

/* Profiling hook: arms three cudaEvent_t handles (any may be NULL) that the
 * NEXT coli_moe_layer_forward call made on this thread records on its
 * stream: `before_experts` just before the gate/up kernel, `after_gateup`
 * between the gate/up and the down kernels, `after_down` after the down
 * kernel.  The events must be created by the caller (with timing enabled);
 * the call consumes the arming.  Always returns COLI_OK. */
coli_status coli_debug_phase_events(void* before_experts, void* after_gateup, void* after_down);

/* Device-side errors of the forward calls made on `workspace` (NULL: the
 * fixed scratch of coli_moe_layer_forward_noalloc on the current device).
 * The first 4 bytes of a workspace are a status word: each
 * coli_moe_layer_forward / coli_moe_stack_forward call clears it when its
 * first kernel starts, and its kernels record the first problem they meet
 * instead of trapping.  This call synchronises `stream`, reads the word and
 * returns COLI_OK (0: no problem), COLI_EDEVICE (1..9: a device-side check
 * failed, e.g. an expert index outside [0, n_experts) in bucketing) or
 * COLI_ETIMEOUT (>= 10: a bounded wait gave up, about a second after the
 * awaited data should have arrived; the kernel then finished without the
 * rest of its work).  coli_last_error() names the code.  The word is left
 * as it is.  COLI_ECUDA if the synchronisation or the read fails. */
coli_status coli_sync_status(void* workspace, void* stream);

/* Test hook for the path above: enqueues one thread that waits on a
 * shared-memory barrier nothing arrives at, for at most `cycles` SM clock
 * cycles (0 .. 4e9), and then records status code 30 in `workspace`'s
 * status word.  No fault and no hang: the wait is bounded. */
coli_status coli_debug_wait_probe(void* workspace, int64_t cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* COLI_H */
