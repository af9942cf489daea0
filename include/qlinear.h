/*
 * qlinear.h -- C ABI of libqlinear.so: quantized decoder projections on B200
 * (sm_100a), Y = (s_x (x) s_w) . (Q(X) . W_q^T).
 *
 * Three schemes, as the model pages define them:
 *   QL_W8A8_INT8_ROW      "Llama 3.1 8B Instruct W8A8", intro and "Loading":
 *                         int8 weights with a bf16 scale for each output row,
 *                         activations quantized to int8 per token, the int8
 *                         products accumulated in int32.
 *   QL_FP8_E4M3_ROW       "Meta-Llama-3.1-8B-Instruct-FP8-dynamic" README,
 *                         "Model Optimizations" and the "Creation" recipe: E4M3
 *                         weights per output channel (static, symmetric), E4M3
 *                         activations per token (dynamic, symmetric).
 *   QL_FP8_E4M3_BLOCK128  "Qwen3 8B FP8", intro and "Loading": E4M3 weights with
 *                         a multiplying scale for each 128x128 block,
 *                         activations quantized to E4M3 in groups of 128 along
 *                         K; widths must be multiples of 128.
 *
 * Numerics (identical in every entry point):
 *   activation scale  s = absmax / 127 (int8) or absmax / 448 (E4M3), one IEEE
 *                     f32 division over the token (row schemes) or over each
 *                     128-wide group of the token (block scheme); an all-zero
 *                     token or group gets s = 0 and codes 0.
 *   activation code   q = clamp(rne(x / s), -127, 127) for int8, or the E4M3
 *                     value nearest x / s (ties to even, saturating at +-448);
 *                     x / s is an IEEE f32 division.
 *   weight scale      int8: bf16(absmax_row / 127); E4M3 row: absmax_row / 448;
 *                     E4M3 block: absmax_block / 448 (f32), block = 128 output
 *                     rows x 128 input columns.
 *   epilogue          row schemes: y = bf16_rne(((f32)acc * s_x[m]) * s_w[n]),
 *                     acc the int32 (int8) or f32 (E4M3) sum over K; block
 *                     scheme: y = bf16_rne(sum_kb P_kb * s_x[m,kb] * s_w[n/128,kb])
 *                     with P_kb the f32 sum over the kb-th 128 inputs.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must be device (or managed) memory of the
 *     current CUDA device; "host" pointers are ordinary host memory.  The
 *     caller owns every buffer; the library never allocates, frees or keeps a
 *     pointer after the call returns.
 *   - bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *   - All matrices are row-major and dense: X / q_x [M,K], W / W_q [N,K]
 *     (nn.Linear [out, in]), Y [M,N]; row scales s_x [M], s_w [N]; block
 *     scales s_x [M, K/128], s_w [N/128, K/128].
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: argument errors are returned before anything is
 *     launched; launch errors come back as QL_ERR_CUDA; faults inside a kernel
 *     surface at the caller's next synchronisation.  No entry point
 *     synchronises except qlinear_get_device_status.
 *   - Preconditions checked on the host: non-null pointers (unless said
 *     optional), M >= 0 (M = 0 is a no-op), N > 0, K > 0, K % 16 == 0, every
 *     device pointer 16-byte aligned, N % 128 == 0 and K % 128 == 0 for the
 *     block scheme, K <= 133144 for int8 (int32 range of K * 127^2) and
 *     K < 131072 for E4M3; M >= 1 with no upper limit except int32 indexing
 *     (M * K and M * N below 2^31).
 *   - The products and the activation quantization are launched with
 *     programmatic dependent launch: a call's kernel may start while the
 *     previous kernel on the stream is finishing.  It reads W_q (and, in the
 *     GEMV, s_w) before it waits for that kernel, and everything else after.
 *     So W_q and s_w must not be written by work still in flight on the same
 *     stream (weights are written once, before the projections run).
 *   - Kernels that wait on a barrier wait a bounded time; if a wait gives up
 *     the kernel records QL_ERR_TIMEOUT in a device status word and returns
 *     without finishing its output.  qlinear_get_device_status reads it.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ql_scheme {
  QL_W8A8_INT8_ROW = 0,
  QL_FP8_E4M3_ROW = 1,
  QL_FP8_E4M3_BLOCK128 = 2
} ql_scheme;

typedef enum ql_status {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1,       /* null pointer, bad scheme, negative size        */
  QL_ERR_UNSUPPORTED_SHAPE = 2, /* a size the scheme or the entry point excludes  */
  QL_ERR_MISALIGNED = 3,        /* a device pointer not 16-byte aligned           */
  QL_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed            */
  QL_ERR_TIMEOUT = 5,           /* a kernel's bounded wait gave up                */
  QL_ERR_DEVICE = 6,            /* no usable sm_100 device is current             */
  QL_ERR_WORKSPACE = 7          /* workspace missing or smaller than required     */
} ql_status;

/* Optional capture of intermediate values for bit-exact checks; pass NULL in
 * production.  Each member may be NULL.  All are device pointers, 16-byte
 * aligned, owned by the caller. */
typedef struct ql_debug {
  void* qx;         /* [M,K] bytes: the activation codes the kernel multiplied */
  float* sx;        /* [M] or [M,K/128]: the activation scales it used        */
  int32_t* acc_i32; /* [M,N]: int32 accumulators before the epilogue (int8)   */
  float* acc_f32;   /* [M,N]: f32 accumulators before the epilogue (E4M3 row) */
} ql_debug;

/* ---------------------------------------------------------------------- */

/* Weight quantization (offline, checkpoint side), on the GPU.
 * Pages: W8A8 intro (int8, a bf16 scale for each output row); FP8-dynamic README
 * "Model Optimizations" / recipe (E4M3, per channel, static, symmetric); Qwen3
 * FP8 intro (E4M3, one multiplier per 128x128 block).
 *   w    device, bf16 [N,K]
 *   wq   device, out: [N,K] int8 or E4M3 bytes
 *   sw   device, out: f32 [N] (row schemes; the int8 scale holds a bf16 value)
 *        or [N/128, K/128] (block scheme)
 * Errors: argument checks as above. */
ql_status qlinear_quantize_weight(ql_scheme scheme, const uint16_t* w, int64_t N, int64_t K,
                                  void* wq, float* sw, void* stream);

/* Dynamic activation quantization (a per-token or per-128-group absmax by warp
 * shuffles, the scale, the rounded codes).  Pages: W8A8 intro and "Loading"
 * (int8 per token); FP8-dynamic recipe (per token, dynamic, symmetric); Qwen3
 * FP8 "Loading" (E4M3 in groups of 128 along K).
 *   x    device, bf16 [M,K]
 *   qx   device, out: [M,K] codes
 *   sx   device, out: f32 [M] (row schemes) or [M, K/128] (block scheme) */
ql_status qlinear_quantize_act(ql_scheme scheme, const uint16_t* x, int64_t M, int64_t K,
                               void* qx, float* sx, void* stream);

/* M = 1 decode product, activation quantization fused: one kernel streams
 * each weight byte once.  Pages: W8A8 "Loading" (a single token takes a
 * kernel that touches every weight byte once); Qwen3 FP8 "Loading" (same, FP8).
 *   x    device, bf16 [1,K]
 *   wq   device, [N,K] codes from qlinear_quantize_weight (or a checkpoint)
 *   sw   device, weight scales as produced by qlinear_quantize_weight
 *   y    device, out: bf16 [1,N]
 *   dbg  optional (NULL): captures q_x, s_x and, for int8, acc_i32 / for E4M3
 *        row, acc_f32 ([1,N]) */
ql_status qlinear_gemv(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                       int64_t N, int64_t K, uint16_t* y, const ql_debug* dbg, void* stream);

/* Several M = 1 products with the same K in one launch: each product keeps
 * its own input, weights, scales and output (e.g. a layer's q, k and v
 * projections of one normalised input, or gate and up), and the numerics of
 * each are those of qlinear_gemv, bit for bit.  Pages: the same as
 * qlinear_gemv (W8A8 and Qwen3 FP8 "Loading": one row in a kernel that reads
 * each weight byte once); a decode step runs a layer's projections that read
 * one input side by side (W8A8 "Against bf16": decoding under CUDA graphs).
 * The SMs are shared out in proportion to the products' weight bytes, each
 * CTA streaming one product.
 *   problems  host array of `count` descriptors, 1 <= count <=
 *             QL_GEMV_MAX_GROUP (read during the call only):
 *               x   device, bf16 [1,K] (products may share one x); or NULL
 *                   when the input comes already quantized:
 *               qx, sx  device, the input's codes [1,K] and scales ([1] or
 *                   [K/128]) as qlinear_quantize_act (or a producer kernel)
 *                   writes them; ignored when x is set
 *               wq  device, [N,K] codes;  sw  device, the matching scales
 *               y   device, out: bf16 [1,N] (outputs must not overlap)
 *               N   output rows (> 0; a multiple of 128 for the block scheme)
 * Errors: argument checks as for qlinear_gemv on every product; count outside
 * [1, QL_GEMV_MAX_GROUP] -> QL_ERR_INVALID_ARG. */
#define QL_GEMV_MAX_GROUP 8
typedef struct ql_gemv_problem {
  const uint16_t* x;
  const void* qx;
  const float* sx;
  const void* wq;
  const float* sw;
  uint16_t* y;
  int64_t N;
} ql_gemv_problem;

ql_status qlinear_gemv_grouped(ql_scheme scheme, const ql_gemv_problem* problems, int count,
                               int64_t K, void* stream);

/* M = 1 product on an input that its producer has already quantized (the
 * activation quantization moved out of the product's critical path: the
 * pages blame the prompt's "two kernels a projection" for its lost time,
 * "Llama 3.1 8B Instruct W8A8", "Against bf16", and the Red Hat W8A8 post
 * the inter-token latency lost to dynamic activation quantization).  The
 * kernel reads the codes and scales instead of quantizing x; everything else
 * is qlinear_gemv, and its output equals qlinear_gemv's on the x those codes
 * came from.
 *   qx  device, [1,K] codes;  sx  device, f32 [1] (row schemes) or [K/128]
 *   wq, sw, y, N, K as for qlinear_gemv
 * Errors: as for qlinear_gemv. */
ql_status qlinear_gemv_prequant(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                                const float* sw, int64_t N, int64_t K, uint16_t* y, void* stream);

/* M = 1 weight-only product ("equivalent" numerics: W8A16 / FP8 weight-only):
 * the activations are not rounded, only the weights are quantized,
 *   y[n] = bf16_rne( sum_k x[k] * (q_w[n,k] * s_w) ),
 * s_w = s_w[n] (row schemes) or s_w[n/128, k/128] (block scheme).  Pages: the
 * W8A8 and Qwen3 FP8 model pages, "Against bf16" (a loader option that never
 * rounds the input); the W8A8 page's "Context" (W8A16 quantizes only the
 * weights and keeps computing in bf16).  One kernel streams each weight byte
 * once, as qlinear_gemv does.
 *   x    device, bf16 [1,K]
 *   wq   device, [N,K] codes from qlinear_quantize_weight (or a checkpoint)
 *   sw   device, the matching weight scales
 *   y    device, out: bf16 [1,N]
 * Arithmetic: x is staged as x * 2^e in f16 (e the power of two that puts the
 * token's absmax in [2^14, 2^15); every element within 2^31 of the absmax is
 * carried exactly), the codes convert exactly to f16, the products are exact
 * and summed in f32 on the tensor cores, then scaled by 2^-e and s_w in f32.
 * Tolerance against the exact value: |y - y_exact| <= 2^-7 |y_exact| + 1e-3.
 * Errors: argument checks as above; K <= 16384 (else QL_ERR_UNSUPPORTED_SHAPE:
 * the staged f16 x takes 2K bytes of shared memory beside the weight ring). */
ql_status qlinear_gemv_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                   const float* sw, int64_t N, int64_t K, uint16_t* y,
                                   void* stream);

/* Weight-only product for 1 <= M <= 32 tokens (the numerics of
 * qlinear_gemv_weight_only, token by token: x not rounded, f32 sums, then the
 * weight scale; tolerance |y - y_exact| <= 2^-7 |y_exact| + 1e-3).  Same
 * pages as qlinear_gemv_weight_only; the W8A8 and Qwen3 FP8 pages run up to
 * 32 tokens on the tensor cores ("Loading").  Up to four tokens ride on the
 * weight-only GEMV kernel's spare MMA columns (K up to 16384 for one or two
 * tokens, 8192 for three or four: the staged f16 tokens and two weight
 * stages must fit the shared memory); other shapes run on the tensor
 * cores (tcgen05 kind::f16: the codes are converted exactly to bf16 in
 * shared memory and multiplied with the bf16 x, K split across the SMs).
 *   x          device, bf16 [M,K];  y  device, out: bf16 [M,N]
 *   workspace  device, qlinear_weight_only_workspace_bytes(scheme, M, N, K)
 *              bytes (0: none needed, NULL allowed), 256-byte aligned,
 *              ZERO-FILLED before its first use; a completed call leaves it
 *              ready for the next call of the same shape (as for
 *              qlinear_gemm_small).  Calls in flight together must not share it.
 * Errors: argument checks as above; M = 0 is a no-op; M > 32 ->
 * QL_ERR_UNSUPPORTED_SHAPE; a missing or small workspace -> QL_ERR_WORKSPACE. */
ql_status qlinear_forward_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                      const float* sw, int64_t M, int64_t N, int64_t K,
                                      uint16_t* y, void* workspace, size_t ws_bytes, void* stream);
size_t qlinear_weight_only_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K);

/* 1 <= M <= 32 product on the tensor cores (tcgen05, tokens on the MMA N side,
 * weights on the 128-row side, K split across the SMs).  Up to four tokens
 * (K <= 16384 for two, K <= 8192 for three or four) run instead on the
 * qlinear_gemv kernel, which carries them on its MMA's spare columns at the
 * weight traffic of one token; the result is the same.  Five to eight tokens
 * with K <= 8192 on at most 8 MiB of weights (a k_proj-sized product) run on
 * that kernel too, as two products of tokens 0-3 and 4..M-1 over the same
 * weights in one launch, unless `dbg` asks for captures (the tensor-core
 * kernel then runs).  Pages: W8A8
 * "Loading" (batches of at most 32 tokens on the tensor cores); Qwen3 FP8
 * "Loading" (same).
 * Activation quantization runs in the same call (a short quantize pass
 * overlapped with the weight stream by programmatic dependent launch).
 *   x          device, bf16 [M,K]
 *   workspace  device, at least qlinear_workspace_bytes(scheme, M, N, K)
 *              bytes, 256-byte aligned, ZERO-FILLED before its first use.
 *              Its leading part (split-tile partial sums and arrival
 *              counters) must be zero when a call starts; a call that
 *              completes leaves it ready for the next call of the same shape,
 *              so one workspace serves call after call of one shape.  Zero it
 *              again before a call of another (M, N, K) or after a
 *              QL_ERR_TIMEOUT.  Two calls in flight at the same time
 *              must not share a workspace.
 *   dbg        optional (NULL): q_x, s_x, acc_i32 (int8) / acc_f32 (E4M3 row) */
ql_status qlinear_gemm_small(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                             int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                             size_t ws_bytes, const ql_debug* dbg, void* stream);

/* qlinear_gemm_small on an input its producer has already quantized (no
 * quantization launch in the call: one kernel per projection; pages as for
 * qlinear_gemv_prequant).  The tensor-core path runs for every 1 <= M <= 32.
 *   qx, sx     device, [M,K] codes and f32 scales ([M] or [M,K/128]) as
 *              qlinear_quantize_act writes them
 *   workspace  as for qlinear_gemm_small (the same size; its quantized-token
 *              part is not used)
 * The output equals qlinear_gemm_small's on the x those codes came from (for
 * int8 bit for bit; E4M3 sums of split tiles may differ in the last bits with
 * the order in which their parts are added, within the output tolerance).
 * Errors: as for qlinear_gemm_small. */
ql_status qlinear_gemm_small_prequant(ql_scheme scheme, const void* qx, const float* sx,
                                      const void* wq, const float* sw, int64_t M, int64_t N,
                                      int64_t K, uint16_t* y, void* workspace, size_t ws_bytes,
                                      void* stream);

/* Large-M product on pre-quantized activations (tcgen05 kind::i8 into int32
 * TMEM accumulators, or kind::f8f6f4 E4M3 into f32; TMA-fed shared-memory
 * ring; the scale epilogue fused; for the block scheme each 128-wide K block
 * is promoted into f32 registers with its two scales).  Pages: W8A8 "Loading"
 * (larger batches: per-token int8 activations, int8 products, int32
 * accumulation); Qwen3 FP8 "Loading" (block scales).
 *   qx, sx     device, from qlinear_quantize_act
 *   workspace  optional (NULL / 0 bytes: whole tiles).  When the output
 *              tiles are few -- 128x256 tiles filling at most half the SMs
 *              with K >= 8192 (e.g. M = 512, N = 4096, K = 14336; every
 *              scheme), or, block scheme, 128x128 tiles filling at most a
 *              quarter of them (e.g. M = 512, N = 1024) -- a workspace of at
 *              least qlinear_workspace_bytes(...) bytes (256-byte aligned,
 *              ZERO-FILLED before its first use) lets the call split each
 *              tile's K blocks over 2 (or, for 128-wide block tiles, up to 4)
 *              CTAs that park their partial sums in it (the block scheme's
 *              f32 running sums; the row schemes' raw s32 / f32
 *              accumulators, added before the scales: int8 outputs stay
 *              bit-exact) -- one 128x256 slab per part per output tile, then
 *              one arrival counter per tile; the last to arrive adds the
 *              parts in part order (the same bits whatever the order of
 *              arrival).  A completed call leaves the counters zero again,
 *              for any next shape; zero the workspace again after a
 *              QL_ERR_TIMEOUT.  Two calls in flight at the same time must not
 *              share it.  qlinear_workspace_bytes returns 0 for shapes that
 *              run whole tiles.
 *   dbg        optional (NULL): acc_i32 (int8) / acc_f32 (E4M3 row) [M,N] */
ql_status qlinear_gemm(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                       const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                       void* workspace, size_t ws_bytes, const ql_debug* dbg, void* stream);

/* qlinear_gemm (block scheme) whose epilogue also quantizes its own output
 * for the product that reads it next: the E4M3 codes of y and one f32 scale
 * per token per 128 outputs, exactly what qlinear_quantize_act writes for
 * the bf16 y (s = absmax / 448 over the 128 bf16 outputs, one IEEE division;
 * code = E4M3(y / s)).  A 128-wide output group lies inside one output tile,
 * so no cross-tile reduction is needed, and the next product runs without a
 * quantization launch of its own ("Llama 3.1 8B Instruct W8A8", "Against
 * bf16": "two kernels a projection"; "Qwen3 8B FP8", "Loading": activations
 * in groups of 128).
 *   y       device, out: bf16 [M,N], or NULL to write only the codes
 *   qy      device, out: [M,N] E4M3 codes
 *   sy      device, out: f32 [M, N/128]
 *   other arguments as for qlinear_gemm
 * Errors: as for qlinear_gemm; a row scheme -> QL_ERR_UNSUPPORTED_SHAPE (its
 * per-token scale spans every output tile). */
ql_status qlinear_gemm_quant_out(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                                 const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                 void* qy, float* sy, void* workspace, size_t ws_bytes,
                                 void* stream);

/* Several large-M products on one pre-quantized input in one launch: each
 * product keeps its own weights, scales and output, and the output tiles of
 * all of them are dealt to the same persistent CTAs, so that products too
 * small to fill the SMs alone (a layer's k and v projections at M = 512) fill
 * them together with their neighbours, and a layer's q, k, v (or gate, up)
 * cost one launch and one quantization of their shared input.  Pages: as for
 * qlinear_gemm (the projections of one decoder layer that read one input).
 * Numerics of each product as qlinear_gemm: int8 bit for bit; E4M3 bit for
 * bit whenever neither call splits K (the block scheme's K split is planned
 * on the group's tile count).
 *   qx, sx     device, the shared input from qlinear_quantize_act
 *   problems   host array of `count` descriptors, 1 <= count <=
 *              QL_GEMM_MAX_GROUP (read during the call only):
 *                wq  device, [N,K] codes;  sw  device, the matching scales
 *                y   device, out: bf16 [M,N] (outputs must not overlap)
 *                qy, sy  NULL, or (block scheme, set for every product of
 *                    the call) device outputs as for qlinear_gemm_quant_out:
 *                    y's E4M3 codes [M,N] and per-128 scales [M,N/128]; y may
 *                    then be NULL
 *                N   output rows (> 0; a multiple of 128 for the block scheme)
 *   workspace  optional, as for qlinear_gemm, of at least
 *              qlinear_gemm_grouped_workspace_bytes(...) bytes
 * Errors: argument checks as for qlinear_gemm on every product; count outside
 * [1, QL_GEMM_MAX_GROUP], qy without sy (or the reverse), codes asked of some
 * products but not all, or no output at all -> QL_ERR_INVALID_ARG; codes
 * with a row scheme -> QL_ERR_UNSUPPORTED_SHAPE. */
#define QL_GEMM_MAX_GROUP 4
typedef struct ql_gemm_problem {
  const void* wq;
  const float* sw;
  uint16_t* y;
  void* qy;
  float* sy;
  int64_t N;
} ql_gemm_problem;

ql_status qlinear_gemm_grouped(ql_scheme scheme, const void* qx, const float* sx,
                               const ql_gemm_problem* problems, int count, int64_t M, int64_t K,
                               void* workspace, size_t ws_bytes, void* stream);
/* Workspace size (bytes) for qlinear_gemm_grouped; Ns: host array of the
 * `count` products' N.  0 means none is needed. */
size_t qlinear_gemm_grouped_workspace_bytes(ql_scheme scheme, const int64_t* Ns, int count, int64_t M,
                                            int64_t K);

/* Several 1 <= M <= 32 products on the same tokens in one launch (a layer's
 * q, k, v, or gate, up, in a small decode batch): the tokens are quantized
 * once, and the 128-row weight tiles of every product share the SM-balanced
 * K split, so that the small products (k and v: 4 MB of weights each) do not
 * pay a launch and a reduction of their own.  Up to four tokens within the
 * GEMV's K limits, and five to eight on at most 8 MiB of weights in all (as
 * for qlinear_gemm_small), run as one grouped GEMV launch instead.  Numerics of each product as qlinear_gemm_small.  Pages: as for
 * qlinear_gemm_small.
 *   x          device, bf16 [M,K] tokens, quantized in the call; or NULL with
 *   qx, sx     device, the tokens already quantized (codes [M,K], scales as
 *              qlinear_quantize_act writes them): the tensor-core kernel runs
 *              for every M, with no quantization launch
 *   problems   host array of `count` descriptors, 1 <= count <=
 *              QL_GEMM_MAX_GROUP (read during the call only): wq, sw, y, N as
 *              for qlinear_gemm_grouped; qy and sy must be NULL
 *   workspace  device, at least qlinear_gemm_small_grouped_workspace_bytes(...)
 *              bytes, 256-byte aligned, zero-filled before its first use (as
 *              for qlinear_gemm_small: a completed call leaves it ready)
 * Errors: as for qlinear_gemm_small on every product; count outside
 * [1, QL_GEMM_MAX_GROUP] or qy / sy set -> QL_ERR_INVALID_ARG. */
ql_status qlinear_gemm_small_grouped(ql_scheme scheme, const uint16_t* x, const void* qx, const float* sx,
                                     const ql_gemm_problem* problems, int count, int64_t M, int64_t K,
                                     void* workspace, size_t ws_bytes, void* stream);
size_t qlinear_gemm_small_grouped_workspace_bytes(ql_scheme scheme, const int64_t* Ns, int count, int64_t M,
                                                  int64_t K);

/* The projection as a model calls it: bf16 X in, bf16 Y out, dispatching on
 * the token count the way the pages' "Loading" sections describe: M = 1 ->
 * qlinear_gemv, 2..32 -> qlinear_gemm_small, > 32 -> qlinear_quantize_act
 * into the workspace, then qlinear_gemm.
 *   workspace  device, qlinear_forward_workspace_bytes(scheme, M, N, K) bytes,
 *              zero-filled before first use (as for qlinear_gemm_small). */
ql_status qlinear_forward(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                          int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                          size_t ws_bytes, void* stream);

/* Workspace sizes (bytes) for the current device; 0 means none is needed.
 * qlinear_workspace_bytes covers qlinear_gemm_small (2 <= M <= 32) and
 * qlinear_gemm (M > 32); qlinear_forward_workspace_bytes adds the quantized
 * activations qlinear_forward keeps there for M > 32. */
size_t qlinear_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K);
size_t qlinear_forward_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K);

/* Test hook for the timeout path (no counterpart in the pages): qlinear_gemv
 * with its weight-copy engine held back, so that every consumer's bounded wait
 * runs out after about 2 s; the kernel records QL_ERR_TIMEOUT (detail: the
 * GEMV's kernel id << 8 | wait site) and returns without writing y.  The
 * context stays usable.  Arguments as for qlinear_gemv. */
ql_status qlinear_debug_gemv_stalled(ql_scheme scheme, const uint16_t* x, const void* wq,
                                     const float* sw, int64_t N, int64_t K, uint16_t* y,
                                     void* stream);

/* Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait gives up.  Returns QL_OK, QL_ERR_TIMEOUT
 * (with *detail, if non-NULL, naming the kernel and the wait site), or
 * QL_ERR_CUDA if the synchronisation itself failed. */
ql_status qlinear_get_device_status(void* stream, uint32_t* detail);

/* Static description of a status code. */
const char* qlinear_status_string(ql_status status);

/* The CUDA error text behind the most recent QL_ERR_CUDA on this thread (and
 * the reason for a QL_ERR_WORKSPACE from qlinear_gemm_small_noalloc). */
const char* qlinear_last_cuda_error(void);

/* qlinear_gemm_small without a caller-provided workspace.  The pages have no
 * counterpart to this entry point: it exists for callers that cannot allocate
 * device memory themselves -- plugin code inside a host framework that has
 * reserved all device memory up front and hands out no allocator, a C caller
 * with nowhere to keep a workspace pointer between calls, or a latency-
 * critical path where cudaMalloc could stall or synchronise the device.
 *
 * The scratch (quantized tokens, split-tile sums and counters) is
 * a fixed 8 MiB array in device global memory that the library declares at
 * file scope; every GPU that loads the library holds it until the process
 * exits.  This call allocates nothing and calls no allocating routine.
 *   - Arguments, layouts, numerics and the 1 <= M <= 32 limit are those of
 *     qlinear_gemm_small; the result is the same.
 *   - A shape whose scratch need (qlinear_workspace_bytes) exceeds 8 MiB is
 *     rejected with QL_ERR_WORKSPACE before anything is launched, and
 *     qlinear_last_cuda_error() says how much it needed.  Every Llama-3.1-8B
 *     and Qwen3-8B projection shape fits at M <= 32 on a 148-SM B200.
 *   - The first call on each device looks up the array's device address with
 *     that device current (a one-time set-up); make that first call before
 *     any stream capture.
 *   - All calls share the one array and it keeps the previous call's
 *     contents: each call clears the sums and counters that must start at zero (an
 *     asynchronous memset on `stream`; none when the shape runs on the GEMV
 *     kernel, which uses no scratch).  Calls whose GPU work overlaps --
 *     on different streams, or from different threads -- race on the array
 *     and give wrong results; serialise them. */
ql_status qlinear_gemm_small_noalloc(ql_scheme scheme, const uint16_t* x, const void* wq,
                                     const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
