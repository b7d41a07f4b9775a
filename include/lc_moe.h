/*
 * lc_moe.h -- C ABI of libmoezero.so: the forward pass of a mixture-of-experts layer with
 * zero-computation experts, and its expert-bias update, on NVIDIA B200 (sm_100a).
 *
 * The method is the one of the LongCat-Flash llm-wiki entity page, section 2.1
 * "Zero-Computation Experts":
 *   MoE(x_t) = sum_{i=1}^{N+Z} g_i E_i(x_t)                  (MoE equation)
 * with N FFN experts (ids 0..N-1) and Z zero-computation experts (ids N..N+Z-1) that return
 * their input, E_i(x_t) = x_t. The router picks K experts per token, zero experts included
 * (section 1 core-parameter table: 12 experts per token including zero experts), steered by
 * per-expert biases b_i that the dynamic computation-budget control of section 2.1 updates by
 *   delta_b_i = mu * (K_e/K * 1/N - T_i / (K * T_all)).
 * The gate is a softmax (section 2.3.2, expert-initialisation variance compensation).
 *
 * Readings of what the page leaves open (kept identical in the CPU oracle used by the tests):
 *   - scores s = softmax of the router logits over all N+Z experts;
 *   - selection key = s_i + b_i (bias in score space, selection only);
 *   - the K largest keys in descending order, equal keys to the lower expert index;
 *   - gates g_r = s_sel[r] / sum of the K chosen s (unbiased scores renormalised);
 *   - FFN experts are SwiGLU: H = silu(x Wg^T) * (x Wu^T), Y = H Wd^T;
 *   - bf16 at H, Y and the output; fp32 for logits, scores, gates and the bias arithmetic;
 *   - the bias rule is applied to all N+Z experts.
 *
 * Conventions for every entry point
 *   - Tensors are dense, row-major, on the current CUDA device, 16-byte aligned.
 *     bf16 tensors are passed as raw pointers to 16-bit IEEE bfloat16 values.
 *   - `stream` is a cudaStream_t (NULL: the legacy default stream). Every call only enqueues
 *     work on that stream and returns; nothing is synchronised except by lc_moe_read_status.
 *   - The caller allocates and owns every buffer, including the workspace `ws`. The library
 *     allocates and frees no device or pinned memory.
 *   - `ws` must be zero-filled before its first use. Its first 256 bytes hold the device status
 *     word: kernels OR LC_MOE_DEV_* bits into it instead of trapping, and it stays set until
 *     lc_moe_read_status clears it. The same 256 bytes hold the grouped expert GEMMs' tile
 *     counters (bytes 64 and 128), which each GEMM launch zeroes on the stream before it runs.
 *     Calls that share a workspace must be ordered on one stream.
 *   - Host-side checks run before any launch; a failing check returns a status code and
 *     enqueues nothing. Functions never abort, throw or print.
 *   - Every entry point except lc_moe_read_status can be captured in a CUDA graph once it has
 *     been called on the device outside a capture (the first call sets kernel attributes and
 *     looks up the driver's tensor-map encoder).
 *   - Shape limits (else LC_MOE_ERR_UNSUPPORTED_SHAPE): d and I multiples of 64 and >= 64;
 *     1 <= K <= 32; K <= N+Z <= 2048; N >= 1; Z >= 0; T >= 0; T*K < 2^31. T = 0 is a no-op.
 */
#ifndef LC_MOE_H
#define LC_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LC_MOE_ABI_VERSION 1

/* Shape of one MoE layer call. T tokens of width d; N FFN experts of width I; Z zero experts;
 * K experts picked per token (zero experts included). */
typedef struct lc_moe_shape {
    int32_t T, d, N, Z, K, I;
} lc_moe_shape;

/* Return codes. */
enum {
    LC_MOE_OK = 0,
    LC_MOE_ERR_INVALID_ARG = 1,       /* null pointer where a buffer is required, bad scalar */
    LC_MOE_ERR_UNSUPPORTED_SHAPE = 2, /* outside the shape limits above */
    LC_MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    LC_MOE_ERR_NOT_SM100 = 4,         /* current device is not compute capability 10.0 */
    LC_MOE_ERR_CUDA = 5,              /* a CUDA runtime/driver call or a launch failed */
    LC_MOE_ERR_DEVICE_STATUS = 6,     /* lc_moe_read_status found device status bits set */
    LC_MOE_ERR_TIMEOUT = 7,           /* lc_moe_read_status found a bounded device wait that gave up */
    LC_MOE_ERR_MISALIGNED = 8         /* a pointer is not 16-byte aligned */
};

/* Device status bits (OR-ed into the workspace's status word by the kernels). */
#define LC_MOE_DEV_IDX_RANGE    0x1u  /* an expert index outside [0, N+Z) was read */
#define LC_MOE_DEV_NAN_KEY      0x2u  /* a routing key was NaN (that token's picks are 0..K-1, gates NaN) */
#define LC_MOE_DEV_WAIT_TIMEOUT 0x4u  /* a pipeline wait hit its time limit; the kernel stopped early */
#define LC_MOE_DEV_DUP_PICK     0x8u  /* a token picked the same expert twice */

/* Workspace sizes. `op` selects the entry point the workspace is for. */
enum {
    LC_MOE_OP_FORWARD = 0,   /* lc_moe_forward / lc_moe_forward_timed */
    LC_MOE_OP_ROUTE = 1,     /* lc_moe_route */
    LC_MOE_OP_PERMUTE = 2,   /* lc_moe_permute */
    LC_MOE_OP_STATUS = 3,    /* every other entry point: the status word only (256 bytes) */
    LC_MOE_OP_FORWARD_FP8 = 4  /* lc_moe_forward_fp8 / _timed (0 unless d and I are multiples of 128) */
};

/* Stages of lc_moe_forward, in launch order (lc_moe_forward_timed records one event before
 * each stage and one after the last). */
enum {
    LC_MOE_STAGE_ROUTER_GEMM = 0,  /* router logits, tensor cores */
    LC_MOE_STAGE_TOPK = 1,         /* softmax + biased top-K + expert histogram */
    LC_MOE_STAGE_PERMUTE = 2,      /* counting sort of FFN picks by expert (3 kernels; 1 when T <= 256) */
    LC_MOE_STAGE_GATHER = 3,       /* copy of token rows into expert order */
    LC_MOE_STAGE_GEMM1 = 4,        /* grouped gate/up GEMM with the SwiGLU epilogue */
    LC_MOE_STAGE_GEMM2 = 5,        /* grouped down GEMM */
    LC_MOE_STAGE_COMBINE = 6,      /* gate-weighted sum with the zero-expert identity term */
    LC_MOE_NUM_STAGES = 7
};

int32_t lc_moe_abi_version(void);

/* Static description of a return code (never NULL). */
const char* lc_moe_strerror(int code);

/* Bytes of workspace that entry point `op` needs for shape `s` (0 if the shape is invalid). */
size_t lc_moe_workspace_bytes(const lc_moe_shape* s, int op);

/* Time limit (nanoseconds, per wait) of every bounded device-side wait of later launches from
 * this process. Default 2e9. A wait that runs out sets LC_MOE_DEV_WAIT_TIMEOUT and its kernel
 * returns early with partial results. Values below 1e6 are raised to 1e6. */
void lc_moe_set_wait_limit_ns(uint64_t limit_ns);

/* Clock probe of the grouped expert GEMMs, for measurement. While set, every launch of grouped
 * GEMM 1 (gate/up + SwiGLU) writes, from the first thread of its CTA 0, the global timer (ns) and
 * that SM's cycle counter when the CTA starts its tiles and when it has finished them, to
 * probe[0..3] (start ns, start cycles, end ns, end cycles); grouped GEMM 2 writes probe[4..7].
 * (end cycles - start cycles) / (end ns - start ns) is the SM clock the launch ran at. probe:
 * device memory of 8 uint64 (the caller's, 8-byte aligned), or NULL to stop (the default).
 * Process-wide like the wait limit; each launch overwrites its four values. */
void lc_moe_set_clock_probe(void* probe);

/* Device check of the bounded waits: one CTA runs the pipelines' bounded wait on a barrier phase
 * that nothing completes (role 0, the current limit) and on the phase role 0 would have released
 * (role 1, four times the limit). On a working device role 0 gives up after the limit, sets
 * LC_MOE_DEV_WAIT_TIMEOUT in the status word of `ws` and raises the CTA's abort flag, which ends
 * role 1's wait; the kernel takes about one limit of device time (the default limit is 2 s, so
 * set a short one with lc_moe_set_wait_limit_ns first) and the context stays usable.
 * lc_moe_read_status then returns LC_MOE_ERR_TIMEOUT. ws: status only (LC_MOE_OP_STATUS bytes). */
int lc_moe_check_wait_timeout(void* ws, size_t ws_bytes, void* stream);

/* Test switch of the abort path of the grouped expert GEMMs (no entry point of its own): with the
 * environment variable LC_MOE_DEBUG_GEMM_ABORT_KSTEP=k set when a GEMM is launched, its MMA
 * issuers give up before their k-th k-step as if a pipeline wait had run out. The other roles of
 * each CTA pair then leave through the abort flag or their own bounded waits (about one wait limit
 * of device time), wait for the copies and MMAs they issued, and free TMEM; the status word gets
 * LC_MOE_DEV_WAIT_TIMEOUT and the GEMM outputs are incomplete. Unset in normal use. */

/*
 * lc_moe_forward -- the whole MoE layer (MoE equation, section 2.1).
 *   x      [T, d]   bf16   token activations x_t
 *   wr     [E, d]   bf16   router weight (E = N + Z), logits z = x Wr^T in fp32
 *   bias   [E]      fp32   routing biases b_i (read only)
 *   w13    [N, 2I, d] bf16 FFN expert e: rows 0..I-1 gate projection Wg, rows I..2I-1 up Wu
 *   w2     [N, d, I]  bf16 FFN expert e: down projection Wd
 *   out    [T, d]   bf16   MoE(x_t)
 *   idx    [T, K]   int32  optional (NULL): chosen expert ids in rank order
 *   gate   [T, K]   fp32   optional (NULL): gates in rank order
 *   counts [E]      int32  optional (NULL): ADDED TO with T_i, the picks of each expert
 *   ws     workspace of lc_moe_workspace_bytes(s, LC_MOE_OP_FORWARD) bytes
 * Rows routed to FFN experts are grouped by expert (stable in token order), run through the
 * grouped SwiGLU GEMMs, and combined with the zero-expert term g_r x_t in rank order.
 */
int lc_moe_forward(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                   const void* w13, const void* w2, void* out, int32_t* idx, float* gate,
                   int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/* lc_moe_forward plus timing: `events` holds LC_MOE_NUM_STAGES + 1 cudaEvent_t handles created
 * by the caller; event i is recorded on `stream` before stage i, the last after the combine. */
int lc_moe_forward_timed(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                         const void* w13, const void* w2, void* out, int32_t* idx, float* gate,
                         int32_t* counts, void* ws, size_t ws_bytes, void* stream,
                         void* const* events);

/*
 * lc_moe_route -- router GEMM, softmax, biased top-K and expert histogram (section 2.1 router
 * with biases; section 2.3.2 softmax gate). Used by the bias-control loop.
 *   x [T,d] bf16, wr [E,d] bf16, bias [E] fp32 -> idx [T,K] int32, gate [T,K] fp32;
 *   counts [E] int32 optional, ADDED TO; logits [T,E] fp32 optional (else kept in ws).
 *   ws: lc_moe_workspace_bytes(s, LC_MOE_OP_ROUTE) bytes.
 */
int lc_moe_route(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                 int32_t* idx, float* gate, int32_t* counts, float* logits, void* ws,
                 size_t ws_bytes, void* stream);

/*
 * lc_moe_bias_update -- expert-bias update of the dynamic computation-budget control
 * (section 2.1):  b_i <- b_i + mu * (K_e/(K N) - T_i/(K T_all))  for all E = N + Z experts,
 * as the fp32 operations a = K_e/(K*N), c_i = T_i/(K*T_all), b_i = b_i + mu*(a - c_i), each
 * rounded to nearest once. bias [E] fp32 in place; counts [E] int32 holds T_i; T_all > 0 is the
 * number of tokens the counts cover. reset_counts != 0 zeroes counts after reading them.
 * Needs 1 <= K_e <= K.
 */
int lc_moe_bias_update(float* bias, int32_t* counts, int64_t T_all, int32_t N, int32_t Z,
                       int32_t K, int32_t K_e, float mu, int32_t reset_counts, void* stream);

/* Reads the workspace's device status word (synchronising `stream`), clears it, and stores it in
 * *status_out (may be NULL). Returns LC_MOE_OK if it was zero, LC_MOE_ERR_TIMEOUT if the
 * wait-timeout bit was set, LC_MOE_ERR_DEVICE_STATUS for any other bit. */
int lc_moe_read_status(void* ws, uint32_t* status_out, void* stream);

/* ---- the stages of lc_moe_forward as separate entry points (same kernels) ---------------- */

/* Router logits z [T, E] fp32 = x [T, d] bf16 * wr [E, d]^T (tcgen05 tensor cores, fp32
 * accumulate). ws: status only. */
int lc_moe_router_logits(const lc_moe_shape* s, const void* x, const void* wr, float* logits,
                         void* ws, size_t ws_bytes, void* stream);

/* Softmax over E, top-K of score + bias, renormalised gates, optional histogram (counts added
 * to). logits [T, E] fp32 -> idx [T, K] int32, gate [T, K] fp32. ws: status only. */
int lc_moe_topk(const lc_moe_shape* s, const float* logits, const float* bias, int32_t* idx,
                float* gate, int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/* Expert-count histogram T_i (the T_i of the bias-update equation): counts [n_bins] int32 is
 * ADDED TO with the number of entries of idx [n] equal to each bin. Entries outside
 * [0, n_bins) set LC_MOE_DEV_IDX_RANGE and are skipped. ws: status only. */
int lc_moe_expert_hist(const int32_t* idx, int64_t n, int32_t n_bins, int32_t* counts, void* ws,
                       size_t ws_bytes, void* stream);

/* Grouping of the FFN picks by expert (only picks of FFN experts become rows):
 *   idx [T, K] int32 -> offsets [N+1] int32 (offsets[N] = M rows), row_token [T*K] int32
 *   (first M entries valid: token of each row), pair_row [T, K] int32 (row of pick (t, r), -1 for
 *   a zero-computation expert), x_perm [T*K, d] bf16 (first M rows: x[row_token[row]]).
 * Rows of an expert are in ascending token order. ws: lc_moe_workspace_bytes(s, LC_MOE_OP_PERMUTE).
 * x_perm may be NULL (no row copy). */
int lc_moe_permute(const lc_moe_shape* s, const int32_t* idx, const void* x, int32_t* offsets,
                   int32_t* row_token, int32_t* pair_row, void* x_perm, void* ws, size_t ws_bytes,
                   void* stream);

/* Grouped SwiGLU experts on rows grouped by lc_moe_permute:
 *   x_perm [T*K, d] bf16 and offsets [N+1] -> h [T*K, I] bf16 = silu(X Wg^T) * (X Wu^T),
 *   y [T*K, d] bf16 = h Wd^T, each row with the weights of its expert; rows >= offsets[N] are
 *   not written. ws: status only. */
int lc_moe_expert_ffn(const lc_moe_shape* s, const void* x_perm, const int32_t* offsets,
                      const void* w13, const void* w2, void* h, void* y, void* ws,
                      size_t ws_bytes, void* stream);

/* Combine: out [T, d] bf16 = sum_r gate[t,r] * (pair_row[t,r] >= 0 ? y[pair_row[t,r]] : x[t]),
 * in fp32 in rank order (the zero-computation term g x_t fused). ws: status only. */
int lc_moe_combine(const lc_moe_shape* s, const void* x, const void* y, const float* gate,
                   const int32_t* pair_row, void* out, void* ws, size_t ws_bytes, void* stream);

/* ---- expert parallelism ---------------------------------------------------------------------
 * The pages deploy the layer with its experts spread over GPUs (LongCat-Flash llm-wiki entity
 * page, section 2.2 ScMoE: expert-parallel dispatch and combine; section 5: multi-GPU
 * deployments). With G ranks, rank r holds FFN experts [r N/G, (r+1) N/G). Each rank routes and
 * groups its own tokens (lc_moe_route / lc_moe_permute over all N experts), sends every rank the
 * contiguous slice of its grouped rows that belongs to that rank's experts (an all-to-all; picks
 * of zero-computation experts, E_i(x) = x, stay on their rank), runs the grouped GEMMs of its own
 * experts on the rows it received, returns each output row to its source (the inverse
 * all-to-all) and combines as lc_moe_combine does. The two calls below are the local step
 * between the exchanges; the exchanges themselves are the caller's (NCCL through
 * torch.distributed in the Python binding). */

/* Expert-major order of rows received source-major.
 *   cnt     [G, n_local] int32 (device): rows source rank s sent for local expert e; the rows
 *           arrived ordered by source, then expert, then the source's token order
 *   perm    [m_cap] int32 (device): perm[i] = arrival index of the i-th row in expert-major
 *           order (expert, then source rank, then arrival order); M = sum(cnt) entries written
 *   offsets [n_local + 1] int32 (device): local expert e owns rows [offsets[e], offsets[e+1])
 *   ws      status only (LC_MOE_OP_STATUS bytes); M > m_cap or a negative count sets
 *           LC_MOE_DEV_IDX_RANGE (entries past m_cap are not written).
 * Needs G * n_local <= 2048 (else LC_MOE_ERR_UNSUPPORTED_SHAPE). */
int lc_moe_ep_regroup_plan(const int32_t* cnt, int32_t G, int32_t n_local, int32_t* perm, int64_t m_cap,
                           int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* Row copy through an index map, rows of row_bytes bytes (a multiple of 16; 16-byte aligned):
 *   scatter = 0: dst[i] = src[map[i]]   (gather: received rows into expert-major order)
 *   scatter = 1: dst[map[i]] = src[i]   (scatter: expert outputs back into arrival order)
 * for i < n; map must be a permutation of [0, n) (an entry outside it sets LC_MOE_DEV_IDX_RANGE
 * in the status word of ws and that row is skipped). ws: status only. */
int lc_moe_copy_rows(const void* src, void* dst, const int32_t* map, int64_t n, int32_t row_bytes,
                     int32_t scatter, void* ws, size_t ws_bytes, void* stream);

/* lc_moe_permute_noalloc -- lc_moe_permute for callers that cannot allocate device memory: for
 * example code running inside an engine whose memory planner hands out all device memory up
 * front and refuses later requests, or a caller with no workspace of its own to pass. The paper
 * has no counterpart: this entry point is an interface choice of this library. Same arguments and results
 * as lc_moe_permute, without the workspace: the two grouping tables live in an array inside the
 * library, reserved on every GPU that loads it until the process exits.
 *   - Capacity: ceil(T/256) * N <= 131072 (e.g. T <= 65536 with N = 512); larger shapes return
 *     LC_MOE_ERR_UNSUPPORTED_SHAPE before any launch.
 *   - status: optional device uint32 (NULL: not reported) that receives the LC_MOE_DEV_* bits,
 *     OR-ed in; the caller clears it.
 *   - The first call on a device looks up the array's device address; make that first call
 *     before any stream capture (a lookup that fails is returned as LC_MOE_ERR_CUDA and tried
 *     again by the next call; only a successful one is kept).
 *   - Every call shares the one array: calls that overlap on the GPU (different streams without
 *     ordering, several host threads) race and give wrong groupings. Calls ordered on one stream
 *     are safe; no state is carried from one call to the next.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int lc_moe_permute_noalloc(const lc_moe_shape* s, const int32_t* idx, const void* x,
                           int32_t* offsets, int32_t* row_token, int32_t* pair_row, void* x_perm,
                           uint32_t* status, void* stream);

/* ---- FP8 experts ---------------------------------------------------------------------------
 * Section 5 of the LongCat-Flash llm-wiki entity page (inference and deployment) lists FP8/BF16
 * quantisation and an FP8 deployment on one node, without a scaling scheme. This library's
 * scheme: E4M3 codes (OCP 8-bit floating point: 4 exponent bits, bias 7, 3 mantissa bits, largest
 * finite 448) with one fp32 scale per row, s = amax / 448, x ~ s * code. All three expert
 * projections run on E4M3 tensor-core operands (tcgen05 kind::f8f6f4, fp32 accumulation): the
 * activation rows (token rows of x, rows of H after their bf16 rounding) are quantised per row
 * on the device, the weights once by the caller. Routing, the combine and the zero-computation
 * experts stay as in lc_moe_forward.
 */

/* Row-wise E4M3 quantisation of a bf16 matrix src [rows, cols] (cols a multiple of 8):
 *   scale[r] = max_c |src[r,c]| / 448 (one fp32 division; 1 for an all-zero row),
 *   dst[r,c] = E4M3(src[r,c] / scale[r]) (one fp32 division, round to nearest even, saturating
 *   at +-448). dst [rows, cols] bytes; scale [rows] fp32 (4-byte aligned). Used to prepare the
 * FP8 expert weights (w13 as [N * 2I, d]) and, inside lc_moe_forward_fp8, the token rows. */
int lc_moe_quantize_e4m3(const void* src, int64_t rows, int32_t cols, void* dst, float* scale,
                         void* stream);

/* lc_moe_forward with E4M3 experts:
 *   w13q      [N, 2I, d] E4M3 codes of W13 (as lc_moe_quantize_e4m3 makes them from [N*2I, d])
 *   w13_scale [N, 2I]    fp32 scale of each W13 row (16-byte aligned)
 *   w2q       [N, d, I]  E4M3 codes of W2 (from [N*d, I])
 *   w2_scale  [N, d]     fp32 scale of each W2 row (16-byte aligned)
 * Each token row x_t is quantised the same way (one scale per token) before the gate/up GEMM:
 * G = (sum_k code_x code_g) * s_x * s_g and U likewise, in fp32; H = bf16(silu(G) * U); each H
 * row is quantised (one scale per row) and Y = bf16((sum_j code_h code_w) * s_h * s_w). The
 * rest of the layer is lc_moe_forward's. Needs d and I multiples of 128 (else
 * LC_MOE_ERR_UNSUPPORTED_SHAPE). ws: lc_moe_workspace_bytes(s, LC_MOE_OP_FORWARD_FP8) bytes. */
int lc_moe_forward_fp8(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                       const void* w13q, const float* w13_scale, const void* w2q,
                       const float* w2_scale, void* out, int32_t* idx, float* gate, int32_t* counts,
                       void* ws, size_t ws_bytes, void* stream);

/* lc_moe_forward_fp8 plus the stage events of lc_moe_forward_timed (the gather stage also holds
 * the quantisation of the token rows, the GEMM 2 stage that of the H rows). */
int lc_moe_forward_fp8_timed(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                             const void* w13q, const float* w13_scale, const void* w2q,
                             const float* w2_scale, void* out, int32_t* idx, float* gate,
                             int32_t* counts, void* ws, size_t ws_bytes, void* stream,
                             void* const* events);

#ifdef __cplusplus
}
#endif

#endif /* LC_MOE_H */
