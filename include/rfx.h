/*
 * rfx.h -- C ABI of the B200 (sm_100a) block-quantised MoE FFN library.
 *
 * The operation: the mixture-of-experts feed-forward step of a
 * DeepSeek-V4-Flash-style model over ROCmFPX-style block-quantised weights,
 * for decode (one token) and speculative verify (q <= 8 token columns), plus
 * the router top-k.  Sources, cited by page title and section:
 *
 *  [TZ] taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI MAX+ 上跑到 32 tok/s",
 *       section "ROCmFPX：把 284B 权重压进 128 GB" -- blocks of 32 weights with
 *       low-bit codes and a scale; ROCmFP2 10 B/block (2.50 bit), ROCmFP3
 *       3.50 bit, ROCmFP4 4.25 bit; routed gate/up in FP2, routed down in FP3,
 *       sensitive projections FP4 or higher.
 *  [AI] ainomam.com, "APU 实现 token 自由：AMD Ryzen AI MAX+ 395 跑 DeepSeek V4
 *       Flash，284B 模型跑出 32 tok/s", section "Lucebox 的优化三板斧" -- 256
 *       routed experts + 1 shared, 6 active per layer; in the q=4 verify path
 *       every packed weight is decoded once and applied to all verify columns;
 *       tuned TOP-K / ARGSORT routing kernels.
 *  [MZ] m.mzlw.cn, "Lucebox专攻DeepSeek V4：DSpark草稿模型、MoE专家并行与
 *       ROCmFPX量化达成42 tok/s", section "MoE 专家并行" -- 43 MoE layers, 256
 *       routed experts, top-6 plus 1 shared expert; section "DSpark 草稿模型"
 *       -- verify width q2..q5.
 *  [AM] ai-manual.ru, "DeepSeek V4 Flash на AMD Ryzen AI MAX+ 395: как
 *       достичь 32 tok/s локального инференса", section "Технические детали
 *       ROCmFPX" -- the MoE gate (router projection) kept at 8 bits.
 *
 * Conventions
 *  - Every function returns an rfx_status (0 = OK).  No exception crosses the
 *    ABI.  rfx_last_error() gives a thread-local message for the last failure.
 *  - "device" pointers are CUDA global-memory pointers of the current device;
 *    "host" pointers are CPU memory.  All buffers are owned by the caller; the
 *    library never allocates device memory (moe_layer_create allocates only a
 *    small host struct; moe_ffn_forward_static uses a workspace array compiled
 *    into the library).
 *  - Device calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *    default stream).  The return code covers argument validation and launch
 *    errors.  Errors found on the device (expert id out of range, a SwiGLU
 *    intermediate that is not a finite fp32 value, a bounded wait that timed
 *    out) set a flag in the workspace that rfx_ws_status() reads after a sync.
 *
 * Packed weight format (this library's reading: the pages give only the block
 * size and the bytes per block).  W[n][k] = scale[n][k/32] * level(code[n][k]):
 *   RFX_FP2: 2-bit codes, level = c - 1.5  (-1.5 .. 1.5), binary16 scale, 10 B/block
 *   RFX_FP3: 3-bit codes, level = c - 3.5  (-3.5 .. 3.5), binary16 scale, 14 B/block
 *   RFX_FP4: 4-bit codes, level = c - 7.5  (-7.5 .. 7.5), E8M0 scale byte
 *            (value 2^(e-127), 0xFF invalid), 17 B/block
 * Blocks run along k (the reduction dimension) of one output row.  Packed
 * layout: row-groups of 16 rows (rows padded to a multiple of 16 with zero
 * codes and zero scales), each a contiguous stream of chunks of up to 8 tiles
 * (tile = 16 rows x 1 block).  A chunk of nt tiles holds nt*16*codebytes of
 * codes followed by nt*16*scalebytes of scales.  Lane L = 4g+t (g = 0..7,
 * t = 0..3) owns nt*2b bytes of codes (b = bits per code): in a partial chunk
 * (nt < 8) at offset L*nt*2b ("lane-major"); in a full chunk as 32-bit words
 * w = 0 .. 4b-1 with word w at byte ((w/4)*32 + L)*16 + (w%4)*4 ("slab-major",
 * so each 128-bit load of a warp reads 512 contiguous bytes).  Per tile
 * the lane owns 8 "registers" r = 0..7, each two codes (low, high element):
 *   m = r>>2, j = r&3, row = g + 8*(j&1), k0 = 16m + 2t + 8*(j>>1) inside the
 *   block; low = code[row][k0], high = code[row][k0+1].
 * A field of a register is a pair of b-bit slots at bit offset f of the two
 * 16-bit halves of a 32-bit word: low code at bits [f, f+b), high code at
 * [16+f, 16+f+b).
 * Full chunks (8 tiles, "plane" layout: the 8 registers of a tile share one
 * offset, in 8 different words):
 *   FP2: 8 words;  register r of tile b -> word r, f = 2b.
 *   FP4: 16 words; register r of tile b -> word r (b < 4) or 8+r (b >= 4),
 *        f = 4*(b&3).
 *   FP3: 12 words; tiles 0..4: word r, f = 3b; tiles 5, 6: r < 4 -> word 8+r,
 *        f = 3(b-5); r >= 4 -> word 4+r, f = 3(b-2); tile 7: r < 4 -> word 8+r,
 *        f = 6; r >= 4 -> bit i (i = 0..2) of the low code at bit 15 and of the
 *        high code at bit 31 of word 3(r-4)+i.
 * Partial chunks (nt < 8, "tile" layout):
 *   FP2: one word per tile; r at f = 2r.
 *   FP4: two words per tile; word m holds r = 4m+j at f = 4j.
 *   FP3: tiles paired (96 bits per lane per pair, 3 words); pair register
 *        R = 8*(tile&1) + r.  R < 15: word R/5, f = 3(R%5).  R = 15: bit i of
 *        the low code at bit 15 and of the high code at bit 31 of word i.  A
 *        lone last tile (odd nt) is a 48-bit little-endian stream of its 16
 *        codes, code 2r+e (e = 0 low, 1 high) at bits [3(2r+e), +3).
 * Scales of a partial chunk: [g][tile][row g, row g+8], binary16 or E8M0
 * bytes.  Full chunk: E8M0 the same; binary16 the scale of (row g + 8h, tile
 * b) at byte ((b/4)*8 + g)*16 + (b%4)*4 + 2h.
 */
#ifndef RFX_H
#define RFX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RFX_OK = 0,
    RFX_EINVAL = -1,        /* bad argument (null pointer, size, format, code or scale value) */
    RFX_EUNSUPPORTED = -2,  /* valid but outside what this build supports (e.g. q > 8) */
    RFX_ECUDA = -3,         /* a CUDA runtime call or launch failed */
    RFX_EDEVICE = -4,       /* device-side check failed (bad expert id, wait timeout) */
    RFX_ERANGE = -5         /* a SwiGLU intermediate overflowed fp32 (inputs outside the fp32 range) */
} rfx_status;

typedef enum { RFX_FP2 = 2, RFX_FP3 = 3, RFX_FP4 = 4 } rfx_format;

/* Thread-local text of the last non-OK status returned on this thread. */
const char* rfx_last_error(void);

/* ------------------------------------------------------------- format --- */

/*
 * Bytes of the packed form of a [rows][cols] matrix: rows padded up to a
 * multiple of 16, times cols/32 blocks, times the block bytes of the format
 * ([TZ] "ROCmFPX：把 284B 权重压进 128 GB": 32 weights per block, 10 B for
 * ROCmFP2).  Returns 0 for an invalid format, rows < 0 or cols % 32 != 0.
 */
size_t rfx_packed_bytes(rfx_format f, int64_t rows, int64_t cols);

/*
 * Host packer.  codes: host uint8 [rows][cols], each < 2^f.  scales: host
 * [rows][cols/32], uint16 binary16 bits for FP2/FP3 (finite values only),
 * uint8 E8M0 for FP4 (0xFF rejected).  dst: host buffer of at least
 * rfx_packed_bytes(f, rows, cols) bytes.  Returns RFX_EINVAL on any bad value;
 * dst is then unspecified.
 */
int rfx_pack(rfx_format f, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols,
             void* dst, size_t dst_bytes);

/* Host inverse of rfx_pack (codes [rows][cols], scales [rows][cols/32]). */
int rfx_unpack(rfx_format f, const void* src, int64_t rows, int64_t cols, uint8_t* codes, void* scales);

/*
 * Device packer: same layout as rfx_pack with all pointers in device memory
 * (codes [rows][cols] uint8, scales [rows][cols/32]).  Asynchronous on stream.
 * Code and scale values are not checked on the device; a code >= 2^f is
 * reduced modulo 2^f.
 */
int rfx_pack_device(rfx_format f, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols,
                    void* dst, void* stream);

/* ------------------------------------------------------------- router --- */

/*
 * Router top-k with softmax over the selected logits ([AI] "Lucebox 的优化三板斧":
 * TOP-K / ARGSORT routing; [MZ] "MoE 专家并行": top-6 of 256).
 * logits: device fp32 [T][E] row-major (finite).  For each token t: idx[t][0..k)
 * = the k largest logits in descending order, equal values ordered by the
 * lower expert index; w[t][j] = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the
 * k selected.  idx: device int32 [T][k]; w: device fp32 [T][k].
 * Limits: 1 <= E <= 1024, 1 <= k <= min(E, 16), T >= 0 (T = 0 is a no-op).
 */
int moe_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, void* stream);

/*
 * Router projection ahead of the top-k: logits[t][e] = sum_h W[e][h] x[t][h]
 * + bias[e], fp32 accumulation (per element a fixed order: independent of T).
 * The gate that decides the routing is kept at high precision ([AM]
 * "Технические детали ROCmFPX": FP8; [TZ] "ROCmFPX：把 284B 权重压进 128 GB":
 * sensitive projections FP4 or above); this library reads it as bf16.
 * w_router: device bf16 bits [E][H]; bias: device fp32 [E] or NULL; x: device
 * bf16 bits [T][H]; both 16-byte aligned.  logits: device fp32 [T][E].
 * Limits: H % 32 == 0, E >= 1, 0 <= T <= 524280 (T = 0 is a no-op).  One launch
 * (programmatic dependent of the kernel before it: it reads W at once and x
 * only after that kernel has finished).
 */
int moe_router_logits(const void* w_router, const float* bias, const void* x, int T, int H, int E, float* logits,
                      void* stream);

/*
 * moe_router_logits followed by moe_router_topk: logits [T][E], idx [T][k],
 * w [T][k] on the device, the same numbers as the two calls.  T <= 8 (decode /
 * verify): one cooperative launch (every CTA resident; a grid-wide barrier
 * orders the logit stores before one warp per column ranks them), a
 * programmatic dependent of the kernel before it.  T > 8: the two launches.
 * Limits: both calls' (E <= 1024, k <= min(E, 16)).
 */
int moe_router_project_topk(const void* w_router, const float* bias, const void* x, int T, int H, int E, int k,
                            float* logits, int32_t* idx, float* w, void* stream);

/* --------------------------------------------------------------- GEMV --- */

/*
 * y[c][n] = sum_k W[n][k] x[c][k] for c < q, n < N: the quantised mat-vec with
 * in-kernel block dequantisation, every block decoded once for all q columns
 * ([AI] "Lucebox 的优化三板斧": decode once, apply to all verify columns).
 * W: device, packed (rfx_pack layout) [N][K].  x: device [q][K], bf16 bits
 * (x_is_fp32 = 0) or fp32 (x_is_fp32 = 1; then |x| must be < 65504).
 * y: device fp32 [q][N].  Limits: K % 32 == 0, 1 <= q <= 8, N >= 1.
 */
int rfx_gemv_q(rfx_format f, const void* W, int64_t N, int64_t K, const void* x, int x_is_fp32, int q,
               float* y, void* stream);

/* ------------------------------------------------------------ MoE FFN --- */

/*
 * One MoE layer ([MZ] "MoE 专家并行"): E routed experts, each with gate and up
 * [I][H] and down [H][I] packed matrices, and an optional shared expert.  The
 * routed matrices of expert e live at base + e * stride (bytes, multiple of
 * 16, device memory); formats are per matrix kind ([TZ]: FP2 gate/up, FP3
 * down, FP4 shared in the pages' assignment; any format is accepted).
 */
typedef struct {
    int H, I, E, k;
    rfx_format f_gate, f_up, f_down;
    const void* gate; const void* up; const void* down;
    size_t stride_gate, stride_up, stride_down;
    int has_shared;
    rfx_format f_sh_gate, f_sh_up, f_sh_down;
    const void* sh_gate; const void* sh_up; const void* sh_down;
} moe_layer_desc;

typedef struct moe_layer moe_layer;

/* Validate d and make a host-side handle (no device memory). */
int moe_layer_create(const moe_layer_desc* d, moe_layer** out);
void moe_layer_destroy(moe_layer* layer);

/*
 * ROCmFPX MIX ([MZ] "ROCmFPX 量化"): the codebook width is chosen per routed
 * expert from its routing heat (hot experts wider), so experts differ in
 * format and in packed size.  Entry e describes routed expert e: the format
 * of its gate and up matrices (one format for both), the format of its down
 * matrix, and the byte offsets of the three packed matrices from the
 * descriptor's gate, up and down bases (multiples of 16).
 */
typedef struct {
    rfx_format f_gate_up, f_down;
    uint64_t off_gate, off_up, off_down;
} moe_expert_mix;

/*
 * As moe_layer_create, with a format per routed expert: mix is a host array
 * of d->E entries; d's routed formats and strides are ignored (its bases,
 * shapes and shared expert are used as given).  Copies the table to the
 * current CUDA device (E * 32 bytes of device memory, allocated here and
 * freed by moe_layer_destroy; the layer is then used on that device).  Every
 * entry point that takes a layer accepts a MIX layer.  Errors: RFX_EINVAL for
 * a bad format or an unaligned offset, RFX_ECUDA if the copy fails.
 */
int moe_layer_create_mix(const moe_layer_desc* d, const moe_expert_mix* mix, moe_layer** out);

/*
 * Device workspace bytes moe_ffn_forward needs for T token columns (T > 8:
 * the prefill workspace, moe_prefill_workspace_bytes).  The
 * workspace holds counters, the SwiGLU intermediate and per-expert partial
 * outputs; it must be zeroed once (rfx_ws_init) before its first use and may
 * then be reused by successive calls on the same stream.  Calls that overlap
 * on the GPU must use different workspaces.
 */
size_t moe_ffn_workspace_bytes(const moe_layer* layer, int T);
int rfx_ws_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Read and clear the device error flag of a workspace.  Synchronises stream.
 * Returns RFX_OK, RFX_EDEVICE (expert id out of range / a bounded wait timed
 * out) or RFX_ERANGE (a SwiGLU value was not a finite fp32 number).
 */
int rfx_ws_status(void* ws, void* stream);

/*
 * MoE FFN for T token columns ([AI] "Lucebox 的优化三板斧"; [MZ] "MoE 专家并行"):
 *   y[t] = sum_j w[t][j] * down_{e_tj}( silu(gate_{e_tj} x[t]) * up_{e_tj} x[t] )
 *          + down_s( silu(gate_s x[t]) * up_s x[t] )      (shared weight 1)
 * with e_tj = idx[t][j], silu(z) = z / (1 + e^-z).  The experts routed by any
 * column are grouped: each packed block of each union expert is read from HBM
 * and decoded once and applied to every column routed to that expert.
 * x: device bf16 bits [T][H], 16-byte aligned.  idx: device int32 [T][k] in [0, E); an id
 * repeated within a row contributes once per entry (its expert output is
 * computed once and weighted by each of its w), an id out of range sets the
 * device error flag and its entry is skipped.  w: device fp32 [T][k].
 * y: device fp32 [T][H].
 * Numerics: every product level * scale * x is exact and accumulated in fp32;
 * h = silu(g) * u is carried into the down projection as a binary16 hi/lo
 * pair of h * 2^n, n a power-of-two scale per expert and column chosen from
 * max |h|, so any h within the fp32 range is representable to about 2^-22
 * relative.  Column t of a T-column call equals a 1-column call bit for bit.
 * Limits: 1 <= T <= 8 (decode / verify), H % 32 == 0, I % 32 == 0, k <= 8;
 * T == 0 is a no-op (so for every call below that takes T).
 * T > 8 runs moe_ffn_prefill instead (bf16 operands; its own limits and
 * workspace size).
 * One cooperative launch of one CTA per SM (all CTAs resident at once: the
 * down rows of an expert wait, through counters in the workspace, for its
 * gate/up rows, and the combine waits at one grid barrier).  A workspace must
 * not be used by two calls that overlap on the GPU.  After a call that
 * reported a device error through rfx_ws_status, re-initialise the workspace
 * with rfx_ws_init before reuse.
 */
int moe_ffn_forward(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w,
                    float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * The routed step from the router logits ([AI] "Lucebox 的优化三板斧": the
 * top-k routing kernel in front of the expert FFN): moe_router_topk of
 * logits (device fp32 [T][E]) into idx (device int32 [T][k]) and w (device
 * fp32 [T][k]), caller-owned outputs, then moe_ffn_forward; two launches on
 * `stream`.  Arguments, workspace and limits as moe_ffn_forward (T > 8: the
 * prefill path, ws sized by moe_ffn_workspace_bytes).
 */
int moe_ffn_forward_logits(const moe_layer* layer, const void* x, int T, const float* logits, int32_t* idx,
                           float* w, float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * The same step from host buffers: x (bf16 bits [T][H]) and the router
 * logits (fp32 [T][E]) are copied host -> device, moe_router_topk and
 * moe_ffn_forward run, and y (fp32 [T][H]) is copied device -> host (one
 * cudaMemcpyAsync per buffer; the host buffers should be pinned for the
 * copies to be asynchronous).  The two uploads run on a stream the layer
 * makes on first use, into one of two buffer sets used in turn, and `stream`
 * waits for them: a call's uploads overlap the kernels of the call before
 * it.  The kernels and the download run on `stream`; x, the logits and y may
 * be reused once `stream` has synchronised.  For T <= 8 a y in page-locked
 * host memory that the device can address (cudaHostAlloc, cudaHostRegister)
 * receives the decode kernel's stores directly instead of a copy.  Inside a CUDA graph capture
 * everything stays on `stream`.  Calls on one layer are serialised by a lock
 * in the layer.  scratch: device, 256-byte aligned,
 * moe_ffn_host_scratch_bytes(layer, T) bytes, caller-owned, zeroed once with
 * rfx_ws_init before its first use; it holds the moe_ffn_forward workspace
 * first (so rfx_ws_status(scratch) reads its device flag), then the device
 * copies and the routing.  T > 8 runs the prefill path.
 */
size_t moe_ffn_host_scratch_bytes(const moe_layer* layer, int T);
int moe_ffn_forward_host(const moe_layer* layer, const void* x, const float* logits, int T, float* y, void* scratch,
                         size_t scratch_bytes, void* stream);

/*
 * Prefill: the same MoE FFN for many tokens as a grouped GEMM on the tcgen05
 * tensor cores ([AI] "Lucebox 的优化三板斧" and [MZ] "MoE 专家并行" for the
 * layer; the page pair's prefill runs the experts as dense contractions).
 *   y[t] = sum_j w[t][j] * down~_{e_tj}( bf16( silu(gate~ x[t]) * (up~ x[t]) ) )
 *          + the same for the shared expert (weight 1)
 * where M~ is the matrix with every weight rounded once to bf16 (nearest
 * even) from its exact value level * scale, the inner products are
 * accumulated in fp32, and bf16() rounds the SwiGLU output to nearest even.
 * The rows routed to each expert are grouped (expert ascending, inside an
 * expert the entries (t, j) in ascending t*k + j order); every packed block of
 * an expert is read and dequantised into shared memory once per 128-row tile
 * and group of up to 256 of its tokens.  The k + 1 contributions to y[t] are
 * added with fp32 atomics, so their order (and the last bit of y) may vary
 * from run to run.
 * x: device bf16 bits [T][H], 16-byte aligned.  idx: device int32 [T][k] in
 * [0, E) (an id repeated within a row counts twice; an id out of range sets
 * the device error flag and the entry is skipped).  w: device fp32 [T][k].
 * y: device fp32 [T][H], 16-byte aligned (overwritten).  ws: 256-byte
 * aligned, moe_prefill_workspace_bytes(layer, T) bytes; only the error flag
 * word needs zeroing (rfx_ws_init) and calls on one workspace must not
 * overlap on the GPU.  Limits: 1 <= T <= 65536, H % 256 == 0, I % 256 == 0.
 * Six launches on `stream` (grouping, gather, gate/up GEMM, down GEMM); can
 * be captured in a CUDA graph.  Returns RFX_EUNSUPPORTED outside the limits.
 */
size_t moe_prefill_workspace_bytes(const moe_layer* layer, int T);
int moe_ffn_prefill(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w, float* y,
                    void* ws, size_t ws_bytes, void* stream);

/*
 * Prefill at a chosen operand precision (the prefill workload dequantises "to
 * bf16 or fp8" for the tensor cores; the exact variant keeps the decode
 * path's numbers, for a prefill whose result must agree with decode):
 *   RFX_PREFILL_BF16  = moe_ffn_prefill (each weight rounded once to bf16,
 *                       h rounded to bf16);
 *   RFX_PREFILL_EXACT = each weight enters the tensor cores as the bf16 pair
 *                       hi + lo, hi = bf16(w), lo = bf16(w - hi), which is
 *                       w exactly (w = level * scale has at most 15
 *                       significant bits); h enters the down projection as
 *                       h1 + h2, h1 = bf16(h), h2 = bf16(h - h1) (16 bits,
 *                       relative error <= 2^-18).  Gate/up take 2 MMAs per
 *                       k-step and matrix, down 4 (hi h1, hi h2, lo h1,
 *                       lo h2): about 2.7 times the tensor work of bf16.
 *                       Accumulation in fp32.
 * Same arguments, limits and behaviour as moe_ffn_prefill otherwise; the
 * exact variant's workspace also holds the h2 rows
 * (moe_prefill_workspace_bytes_ex).  Unknown precision: 0 bytes /
 * RFX_EINVAL.
 */
#define RFX_PREFILL_BF16 0
#define RFX_PREFILL_EXACT 1
size_t moe_prefill_workspace_bytes_ex(const moe_layer* layer, int T, int precision);
int moe_ffn_prefill_ex(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w, float* y,
                       void* ws, size_t ws_bytes, int precision, void* stream);

/*
 * Device pointers into a prefill workspace after a moe_ffn_prefill call (for
 * inspection and tests): counts[E] tokens per routed expert; row_token and
 * row_weight [routed_rows] the token and combine weight of each grouped row
 * (rows of expert e start at the sum of the counts of the experts below e;
 * only the first sum(counts) rows are defined); h bf16 bits [h_rows][I], the
 * SwiGLU output of every grouped row, then of the shared expert for tokens
 * 0..T-1 (rows routed_rows + t).
 */
typedef struct {
    const int32_t* counts;
    const int32_t* row_token;
    const float* row_weight;
    const void* h;
    int64_t routed_rows;
    int64_t h_rows;
    const void* h_lo;   /* after an exact-precision call: h2 = bf16(h - h1) of every row, same layout as h */
} moe_prefill_ws_view;
int moe_prefill_view(const moe_layer* layer, int T, const void* ws, moe_prefill_ws_view* view);

/*
 * moe_ffn_forward_static -- the same MoE FFN as moe_ffn_forward for callers
 * that cannot allocate device memory (a serving loop with a no-allocation
 * rule, a plugin that does not own the device allocator, a fixed-budget
 * embedded runtime).  The pages have no counterpart: this is a property of
 * the library, not of the method.
 * The workspace is a 16 MiB array compiled into the library (held on every
 * GPU that loads it until the process exits); calls that would need more
 * (moe_ffn_workspace_bytes) return RFX_EUNSUPPORTED.  T > 8 takes the prefill
 * path in the same array, within the same 16 MiB limit.  Each call looks up
 * the array's device address on the current device; the first lookup on a
 * device loads the library's device code there, so make the first call
 * before any stream capture on that device.  All calls on a device share the
 * array: each clears its control words with an asynchronous memset on
 * `stream`, and calls that overlap on the GPU race and give wrong results.
 * Device-side error flags are not reported here (use moe_ffn_forward with
 * your own workspace for that).
 * x, idx, w, y, T and stream as in moe_ffn_forward.  Allocates nothing.
 */
int moe_ffn_forward_static(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w,
                           float* y, void* stream);

/*
 * Layer chaining for a stack of MoE layers (m.mzlw.cn, "Lucebox专攻DeepSeek
 * V4…", section "MoE 专家并行": 43 MoE layers; the chaining rule is this
 * library's stack workload): x_next[t] = bf16(y[t] / sqrt(mean(y[t]^2))),
 * the mean over the H values of column t, computed in fp64 and rounded once
 * to bf16 (nearest even).  y: device fp32 [T][H]; x_next: device bf16 bits
 * [T][H] (may not alias y).  T == 0 is a no-op.
 */
int moe_rms_norm_bf16(const float* y, int T, int H, void* x_next, void* stream);

/*
 * A stack of L layers for T <= 8 token columns, all on `stream`: for l = 0..L-1,
 * (idx, w) = moe_router_topk(logits[l]), y_l = moe_ffn_forward(layer l, x_l),
 * x_{l+1} = moe_rms_norm_bf16(y_l); y receives y_{L-1}.  logits: device fp32
 * [L][T][E]; x: device bf16 bits [T][H] (x_0); y: device fp32 [T][H].  All
 * layers must share H, E and k.  The workspace (moe_stack_workspace_bytes,
 * 256-byte aligned, caller-owned) holds one moe_ffn_forward workspace (zero it
 * once with rfx_ws_init), the routing of every layer and two fp32 activation
 * buffers.  Launches 1 + L kernels: the router for all L * T rows at once,
 * then one MoE FFN kernel per layer; for l > 0 that kernel reads y_{l-1} and
 * applies the unit-RMS bf16 step itself while it stages x (the same bits as
 * moe_rms_norm_bf16).  The result equals the step-by-step calls bit for bit.
 * Can be captured in a CUDA graph.
 */
size_t moe_stack_workspace_bytes(const moe_layer* const* layers, int L, int T);
int moe_stack_forward(const moe_layer* const* layers, int L, const float* logits, const void* x, int T, float* y,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * Test hook for the device error path (no counterpart on the pages).  From the
 * next call on, on every thread: moe_ffn_forward (T <= 8) and moe_ffn_prefill
 * launches give up each bounded wait after wait_cycles SM clocks (0: the
 * default, about 2 s for decode and 0.5 s for prefill), and `fault` plants a
 * wait that cannot end: 1 = the decode kernel's final grid barrier waits for
 * one CTA more than the grid has; 2 = no expert of a decode call ever becomes
 * ready for its down projection; 3 = the prefill down GEMM waits for a unit
 * that is never handed out.  The kernel then sets its timeout flag, drains its
 * copies and returns: rfx_ws_status gives RFX_EDEVICE, and the workspace needs
 * rfx_ws_init before its next use.  fault = 0 restores normal operation.  Not
 * for production use.
 */
int rfx_debug_set_fault(int fault, long long wait_cycles);

#ifdef __cplusplus
}
#endif
#endif /* RFX_H */
