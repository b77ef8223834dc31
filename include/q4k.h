/*
 * q4k.h -- C ABI of the Q4_K weight-only matrix-product library for NVIDIA
 * B200 (sm_100a).
 *
 * The operations are the hot path of GGUF Q4_K inference as the hipEngine
 * 0.3.0 README describes it ("GGUF Support": Q4_K quant readers, the
 * bulk-prefill path; "Quickstart": the WMMA-prefill / GEMV-decode session
 * profile; "Architecture at a glance": the moe kernel family) and as the
 * hipster README's claims table measures it (GEMV GB/s, "MoE grouped GEMM").
 *
 * Q4_K super-block (llama.cpp-style K-quant; 256 weights in 144 bytes):
 *   bytes 0-1   d     IEEE binary16, little-endian
 *   bytes 2-3   dmin  IEEE binary16
 *   bytes 4-15  eight six-bit (sc_j, m_j) pairs:
 *                 j<4 : sc_j = s[j] & 63, m_j = s[j+4] & 63
 *                 j>=4: sc_j = (s[j+4] & 15) | (s[j-4] >> 6) << 4
 *                       m_j  = (s[j+4] >> 4) | (s[j]   >> 6) << 4
 *   bytes 16-143 quants: weight i = 64c + 32h + l is nibble h (0 = low) of
 *                 quant byte 32c + l; it uses pair j = i / 32
 *   w_i = d * sc_j * q_i - dmin * m_j
 * A Q4_K matrix with N rows and K inputs is stored row-major as
 * [N][K/256] blocks, so one row is K/256*144 contiguous bytes.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers (cudaMalloc'd or equivalent),
 *    owned by the caller. The library allocates no device memory, keeps no
 *    per-call state except a device status word, and never synchronises
 *    the stream (except q4k_last_device_status).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call is asynchronous on that stream.
 *  - Activations are bf16 bit patterns (uint16_t), row-major [M][K].
 *    Matmul outputs are fp32 row-major [M][N].
 *  - Base pointers must be 16-byte aligned. K must be a multiple of 256.
 *  - A host-detectable error returns a nonzero q4k_status before anything
 *    is launched and writes nothing. Unsupported shapes fail with
 *    Q4K_ERR_UNSUPPORTED; there is no fallback path.
 *  - Device-side errors (a bounded wait that gave up, an index out of
 *    range) are latched in a device status word that
 *    q4k_last_device_status() reads and clears.
 *  - Results are deterministic: the same inputs give bit-identical outputs
 *    (no floating-point atomics on any result path).
 */
#ifndef Q4K_H
#define Q4K_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  Q4K_OK = 0,
  Q4K_ERR_NULL = 1,           /* a required pointer is NULL                        */
  Q4K_ERR_ALIGN = 2,          /* a pointer is not 16-byte aligned                 */
  Q4K_ERR_SHAPE = 3,          /* a size is negative/zero where not allowed, or
                                 K % 256 != 0                                      */
  Q4K_ERR_UNSUPPORTED = 4,    /* a valid shape outside the supported set           */
  Q4K_ERR_WORKSPACE = 5,      /* workspace missing or smaller than required        */
  Q4K_ERR_LAUNCH = 6,         /* the CUDA launch itself failed                     */
  Q4K_ERR_DEVICE_TIMEOUT = 7, /* a bounded device-side wait gave up                */
  Q4K_ERR_DEVICE_BOUNDS = 8,  /* a device-side index check failed                  */
  Q4K_ERR_CUDA = 9,           /* a CUDA runtime call returned an error             */
  Q4K_ERR_DEVICE_RANGE = 10,  /* a value may not fit the fp16 operands of the
                                 tensor-core grouped path: |x| > 65504, or a
                                 sub-block whose bound 15*|d*sc| + |dmin*m|
                                 exceeds 65504                                     */
  Q4K_ERR_TOO_LARGE = 11      /* the problem needs more than the fixed scratch of
                                 the no-allocation entry point                     */
} q4k_status;

enum { Q4K_ACT_NONE = 0, Q4K_ACT_SWIGLU = 1 };
enum { Q4K_OP_GEMM = 1, Q4K_OP_ROUTE = 2, Q4K_OP_GROUPED = 3, Q4K_OP_GEMV = 4 };

/* Dequantise `nblocks` consecutive Q4_K blocks (hipEngine 0.3.0 README,
 * "GGUF Support": the Q4_K quant reader).
 *   W    [nblocks][144] bytes.
 *   out  out_bf16 == 0: fp32 [nblocks*256], each value RN_fp32 of the exact
 *        d*sc*q - dmin*m (bit-exact);
 *        out_bf16 != 0: bf16 bits [nblocks*256] = RN_bf16 of that fp32 value.
 * nblocks == 0 is a no-op. */
q4k_status q4k_dequant(const void* W, int64_t nblocks, int out_bf16, void* out, void* stream);

/* Decode GEMV, 1 <= M <= 32 tokens (hipEngine 0.3.0 README, "Quickstart":
 * the GEMV-decode half of the WMMA-prefill/GEMV-decode session profile).
 *   Y[m][n] = sum_k w[n][k] * X[m][k],  W [N][K/256] blocks, X bf16 [M][K],
 *   Y fp32 [M][N].  N % 16 == 0.  M == 0 or N == 0 is a no-op.
 *   ws/ws_bytes: device scratch of q4k_workspace_bytes(Q4K_OP_GEMV, M, N, K,
 *   0, 0) bytes (required; some launch shapes leave it untouched). Each
 *   token's activations are taken per 256-wide block, scaled by a power of two
 *   so the block's largest magnitude lands in [2^14, 2^15), and converted to
 *   fp16: exact for every bf16 value within a factor 2^31 of that largest
 *   magnitude (smaller ones keep fp16 subnormal resolution, 2^-24 of the
 *   scaled unit). The 4-bit weights and their six-bit scales enter exactly;
 *   products accumulate in fp32. Calls sharing `ws` must be ordered on one
 *   stream.
 * Within a token class (M = 1..8, 9..16, 17..32) row m of the result does not
 * depend on the other rows of X (bit-identical to any other call of the same
 * class on that row). */
q4k_status q4k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                    void* ws, size_t ws_bytes, void* stream);

/* Decode GEMV over Q5_K weights, the Q4_K_M files' other large tensor family
 * (hipEngine 0.3.0 README, "GGUF Support": the tensor-family table lists Q5_K
 * beside Q4_K). W [N][K/256] Q5_K blocks of 176 bytes: fp16 d, fp16 dmin,
 * the Q4_K 12-byte six-bit (sc, m) packing, 32 bytes qh, 128 bytes of low
 * nibbles in the Q4_K order; weight 64c+32h+l = nibble h of byte 48+32c+l
 * plus 16 x bit 2c+h of qh[l], w = d*sc*q - dmin*m with q in 0..31.
 * Everything else -- X, Y, ws (q4k_workspace_bytes(Q4K_OP_GEMV, ...)), the
 * shapes, errors, the arithmetic and the per-class batch invariance -- as
 * q4k_gemv. */
q4k_status q5k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                    void* ws, size_t ws_bytes, void* stream);

/* Decode GEMV over Q6_K weights, the remaining large tensor family of a Q4_K_M
 * file (hipEngine 0.3.0 README, "GGUF Support": the tensor-family table lists
 * Q6_K beside Q4_K, Q5_K and Q8_0). W [N][K/256] Q6_K blocks of 210 bytes:
 * ql[128] (low four bits), qh[64] (high two bits), 16 signed byte scales, fp16
 * d; weight i = 128n + 32u + l is nibble u/2 of ql[64n + 32(u%2) + l] plus 16 x
 * bits 2u, 2u+1 of qh[32n + l], minus 32; w = d * scale[i/16] * q, q in
 * -32..31. W must be 16-byte aligned (its rows are then 2-byte aligned: 210-byte
 * blocks). The quants enter the tensor-core MMA exactly (q as an fp16 integer),
 * the signed scales and d in fp32. Everything else -- X, Y, ws
 * (q4k_workspace_bytes(Q4K_OP_GEMV, ...)), the shapes, errors and the
 * activation representation -- as q4k_gemv; results are batch-invariant within
 * each token class (1..8, 9..16, 17..32). */
q4k_status q6k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                    void* ws, size_t ws_bytes, void* stream);

/* The Q8 activation lane of the decode GEMV: an opt-in, accuracy-traded form of
 * q4k_gemv (hipster/hipEngine READMEs: the "fast" GEMV lane policy, dp4a route,
 * accuracy traded). Same arguments, workspace, shapes and errors as q4k_gemv.
 * Each token's activations are quantised per 256-wide column: amax = max|x|,
 * d_x = amax/127, q = rint(x * (127/amax)) clamped to +-127 (every step one
 * fp32 operation, round to nearest even); the result is
 *   Y[m][n] = sum_kb d_x[m][kb] * sum_k w[n][k] * q[m][k]
 * with the 4-bit x 8-bit products and their six-bit scaling summed exactly in
 * int32 per super-block (integer tensor-core MMA), the rest in fp32. Its error
 * against q4k_gemv's product is bounded by sum_k |w[n][k]| * |x - d_x*q| (at
 * most half a step d_x/2 per value). Row m does not depend on the other rows of
 * X at any M. */
q4k_status q4k_gemv_q8(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                       void* ws, size_t ws_bytes, void* stream);

/* Decode GEMV over Q8_0 weights (the same tensor-family table lists Q8_0).
 * W [N][K/32] blocks of 34 bytes: fp16 d (little-endian), then 32 two's-
 * complement bytes q; w = d*q. K % 256 == 0 (the GEMV reads eight blocks per
 * 256-wide column). Everything else -- X, Y, ws (q4k_workspace_bytes(
 * Q4K_OP_GEMV, ...)), shapes, errors, the activation pre-pass -- as q4k_gemv;
 * each block's 32 products enter exactly (q + 128 as an fp16 subnormal, the
 * -128 offset through the block's activation sum) and accumulate in fp32.
 * Row m of the result does not depend on the other rows of X at any M. */
q4k_status q80_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                    void* ws, size_t ws_bytes, void* stream);

/* Load-time repack of Q4_K weights for the decode GEMV (hipEngine 0.3.0
 * README, "GGUF Support": the decode-repacked layouts). A byte permutation:
 * the same 144 bytes per super-block, so the same HBM traffic.
 *   Wr[((T*(K/256) + kb)*128 + r)*144 + b] holds super-block kb of weight row
 *   128*T + r (rows are grouped in 128-row tiles; a tile's super-block column
 *   is contiguous). Inside the 144 bytes, bytes 0..15 (d, dmin, scales) are
 *   unchanged and quant byte 32c + 8t + e (chunk c, quarter t, e = 0..7) moves
 *   to 16 + 32t + 8c + e: the eight bytes a GEMV thread takes from each chunk
 *   lie together. Rows past N (up to the next multiple of 128) are zero.
 *   q4k_repacked_bytes(N, K) = ceil(N/128)*128 * K/256 * 144 (0 for a bad
 *   shape). W and Wr are device buffers of the caller, 16-byte aligned, not
 *   overlapping. */
int64_t q4k_repacked_bytes(int N, int K);
q4k_status q4k_repack(const void* W, int N, int K, void* Wr, void* stream);

/* q4k_gemv on repacked weights (same arguments, Wr from q4k_repack with the
 * same N, K): each 128-row tile streams as one contiguous run per super-block
 * column and every thread reads its quant bytes with two 16-byte loads. Same
 * arithmetic in the same order as q4k_gemv: bit-identical results. */
q4k_status q4k_gemv_repacked(const void* Wr, const uint16_t* X, float* Y, int M, int N, int K,
                             void* ws, size_t ws_bytes, void* stream);

/* Prefill GEMM on tcgen05 tensor cores with the Q4_K weights dequantised
 * tile by tile into shared memory (hipEngine 0.3.0 README, "GGUF Support":
 * the bulk-prefill path).
 *   Y[m][n] = sum_k w[n][k] * X[m][k] with w rounded to bf16 (RN of the fp32
 *   dequant), bf16 x bf16 products, fp32 accumulation.
 *   N % 256 == 0, K % 256 == 0, M >= 1 (ragged M handled).
 *   ws/ws_bytes: unused (pass NULL, 0); reserved for split variants. */
q4k_status q4k_gemm(const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                    void* ws, size_t ws_bytes, void* stream);

/* The GEMM half of the unfused chain that q4k_gemm fuses: with the weights first
 * dequantised to bf16 by q4k_dequant(out_bf16 = 1), this multiplies them with
 * exactly q4k_gemm's tiles, tcgen05 MMAs and summation order, so
 *   bf16w_gemm(q4k_dequant(W, bf16), X) == q4k_gemm(W, X)   bit for bit
 * (hipEngine 0.3.0 README, "Core principles": every fused composite has a
 * numerically equivalent unfused chain). Wb bf16 [N][K], X bf16 [M][K], Y fp32
 * [M][N], all row-major; N % 256 == 0, K % 256 == 0; errors as q4k_gemm. */
q4k_status bf16w_gemm(const uint16_t* Wb, const uint16_t* X, float* Y, int M, int N, int K, void* stream);

/* Top-k routing and token permutation for a mixture-of-experts layer
 * (hipEngine 0.3.0 README, "Architecture at a glance": moe kernels).
 *   logits     fp32 [M][E] router logits.
 *   topk_ids   int32 [M][topk]: experts ranked by logit, descending, equal
 *              logits to the lower id.
 *   topk_w     fp32 [M][topk]: softmax over the selected logits.
 *   expert_offsets int32 [E+1]: exclusive prefix sum of per-expert counts.
 *   perm       int32 [M*topk]: sorted row -> flat index t*topk + j, sorted
 *              by (expert, flat index).
 *   inv_perm   int32 [M*topk]: flat index -> sorted row.
 *   row_token  int32 [M*topk]: sorted row -> token.
 *   ws         device scratch of q4k_workspace_bytes(Q4K_OP_ROUTE, M, 0, 0,
 *              E, topk) bytes (per-tile expert histograms).
 * 1 <= E <= 1024, 1 <= topk <= min(E, 16). M == 0 writes expert_offsets
 * as zeros only. */
q4k_status moe_route_permute(const float* logits, int M, int E, int topk,
                             int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                             int32_t* perm, int32_t* inv_perm, int32_t* row_token,
                             void* ws, size_t ws_bytes, void* stream);

/* moe_route_permute without a workspace argument: for callers that cannot
 * allocate device memory at call time -- a runtime whose device memory is
 * owned and budgeted by a host framework that exposes no allocator to this
 * library, or a serving loop that forbids cudaMalloc after start-up because
 * it can synchronise the device and stall other streams. There is no
 * counterpart of this entry point in the paper; it exists only for such callers.
 * Same arguments, results and errors as moe_route_permute, except:
 *  - The per-tile expert histograms live in one fixed device array inside
 *    this library, 65536 int32 (256 KiB), which every GPU that loads the
 *    library keeps until process exit. Problems needing more, i.e.
 *    ceil(M / 32) * E > 65536, return Q4K_ERR_TOO_LARGE and launch nothing.
 *  - The first call on a device looks up that array's device address (a
 *    cudaGetSymbolAddress with the device current); make that first call
 *    before any stream capture on that device.
 *  - Every call, on any stream, uses the same array and it keeps the last
 *    call's contents (each call overwrites every entry it reads, so nothing
 *    needs clearing). Calls that may overlap on the GPU race: order them on
 *    one stream, or with events.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
q4k_status moe_route_permute_noalloc(const float* logits, int M, int E, int topk,
                                     int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                     int32_t* perm, int32_t* inv_perm, int32_t* row_token,
                                     void* stream);

/* Grouped expert matmul over rows sorted by expert (hipster README, claims
 * table: "MoE grouped GEMM"; hipEngine 0.3.0 README, moe kernels).
 *   W_experts  [E][N][K/256] Q4_K blocks.
 *   A          bf16 activations; row r of the sorted order reads
 *              A[row_gather[r]] (row_gather may be NULL: A[r]).
 *   expert_offsets int32 [E+1] (device): rows [off[e], off[e+1]) use expert e.
 *   rows       total rows = off[E] (host value; must match the device array).
 *   max_rows_hint  upper bound on any single expert's row count (for a
 *              top-k layer over M tokens: M). <= 32 selects a decode kernel
 *              with the arithmetic of q4k_gemv at 1..8 tokens: for K <= 5120
 *              the grouped stationary GEMV (no activation pre-pass; any row
 *              count per expert, 8 rows per pass over its weights; each row's
 *              result bit-identical to q4k_gemv of that expert on up to 8 rows;
 *              offsets that are not non-decreasing within [0, rows] latch
 *              Q4K_ERR_DEVICE_BOUNDS and nothing is written), for longer K the
 *              grouped ring GEMV (at most 32 rows per expert, else
 *              Q4K_ERR_DEVICE_BOUNDS is latched);
 *              larger selects the tcgen05 grouped GEMM, whose operands are
 *              fp16: weights RN_fp16 of the fp32 dequant, activations
 *              converted from bf16 (|values| must stay below 65504, else
 *              Q4K_ERR_DEVICE_RANGE is latched).
 *   act == Q4K_ACT_NONE:   out fp32 [rows][N].
 *   act == Q4K_ACT_SWIGLU: out bf16 [rows][N/2], h = SiLU(g) * u with
 *              g = columns 0..N/2-1 (gate rows of W) and u = N/2..N-1 (up rows).
 *   ws/ws_bytes: device scratch of q4k_workspace_bytes(Q4K_OP_GROUPED, rows,
 *              N, K, E, 0) bytes (required when max_rows_hint <= 32, used by the
 *              ring GEMV; may be NULL when max_rows_hint > 32).
 * N % 32 == 0 (SWIGLU: N/2 % 16 == 0), rows == 0 is a no-op. */
q4k_status moe_q4k_grouped(const void* W_experts, int E, int N, int K, const uint16_t* A,
                           const int32_t* row_gather, const int32_t* expert_offsets,
                           int rows, int max_rows_hint, int act, void* out,
                           void* ws, size_t ws_bytes, void* stream);

/* Routing and the grouped gate_up GEMV of the decode MoE layer in one launch
 * (hipEngine 0.3.0 README, "Core principles": the route composite fused with the
 * expert matmul that follows it). Equivalent to
 *   moe_route_permute(logits, M, E, topk, topk_ids, topk_w, expert_offsets, perm,
 *                     inv_perm, row_token, ...)  and then
 *   moe_q4k_grouped(W_gate_up, E, N, K, X, row_gather = row_token, expert_offsets,
 *                   M*topk, M, Q4K_ACT_SWIGLU, h, ...),
 * bit for bit (every CTA of the GEMV routes all tokens with the same code and order
 * as the routing kernel; one writes the routing outputs).
 *   logits fp32 [M][E]; X bf16 [M][K]; W_gate_up Q4_K [E][N][K/256] (gate rows
 *   first, then up rows); h bf16 [M*topk][N/2]; the routing outputs as in
 *   moe_route_permute (all device, caller-owned, written).
 * Supported: 1 <= M <= 32, E <= 256, topk <= 16, 1536 <= K <= 5120 (at least six
 * consumer warps to host the routing warps), N % 32 == 0; anything else returns
 * Q4K_ERR_UNSUPPORTED (use the two calls). No workspace.
 * M == 0 only clears expert_offsets. Device errors as the two calls. */
q4k_status moe_route_gate_up(const float* logits, int M, int E, int topk, int32_t* topk_ids, float* topk_w,
                             int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm, int32_t* row_token,
                             const void* W_gate_up, int N, int K, const uint16_t* X, void* h, void* stream);

/* Weighted combine of the expert outputs back into token order
 * (hipEngine 0.3.0 README, "Core principles": the gate_combine part of the
 * fused gate_combine_residual composite).
 *   y[t][h] = sum_{j=0..topk-1} topk_w[t][j] * O[inv_perm[t*topk + j]][h],
 *   summed in increasing j.  O fp32 [M*topk][H], Y fp32 [M][H].
 * H % 4 == 0.  M == 0 is a no-op. */
q4k_status moe_combine(const float* O, const int32_t* inv_perm, const float* topk_w,
                       int M, int topk, int H, float* Y, void* stream);

/* The combine fused with the residual add (hipEngine 0.3.0 README, "Core
 * principles": the gate_combine_residual composite).
 *   y[t][h] = residual[t][h] + (sum_{j=0..topk-1} topk_w[t][j] * O[inv_perm[t*topk + j]][h]),
 *   the sum taken as in moe_combine, then one fp32 add, so the result equals
 *   moe_combine's followed by an fp32 add of residual, bit for bit.
 * residual fp32 [M][H], caller-owned; it may be the same buffer as Y (in
 * place). Shapes, alignment and errors as moe_combine; a null residual is
 * Q4K_ERR_NULL. */
q4k_status moe_combine_residual(const float* O, const int32_t* inv_perm, const float* topk_w,
                                const float* residual, int M, int topk, int H, float* Y,
                                void* stream);

/* The router product in front of moe_route_permute (the routing front of the
 * fused MoE layer; hipEngine 0.3.0 README, "Architecture at a glance": moe
 * kernels).
 *   logits[t][e] = sum_k X[t][k] * W_router[e][k]: X bf16 [M][H], W_router
 *   bf16 [E][H], logits fp32 [M][E] (caller-owned, written), the bf16
 *   products exact in fp32, summed in fp32 in a fixed order.
 * Then exactly moe_route_permute(logits, ...): the remaining arguments, the
 * workspace and the errors are that call's. H % 8 == 0; M <= 65535. */
q4k_status moe_route_permute_hidden(const uint16_t* X, const uint16_t* W_router, int M, int E, int H,
                                    int topk, float* logits, int32_t* topk_ids, float* topk_w,
                                    int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                                    int32_t* row_token, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace an entry point needs for these sizes
 * (Q4K_OP_ROUTE: moe_route_permute with M tokens and E experts;
 *  Q4K_OP_GEMV: q4k_gemv with M tokens and K inputs;
 *  Q4K_OP_GROUPED: moe_q4k_grouped with M = rows and K inputs;
 *  Q4K_OP_GEMM: 0). */
size_t q4k_workspace_bytes(int op, int M, int N, int K, int E, int topk);

/* Synchronises `stream`, returns the device status word (Q4K_OK if no
 * device-side error was latched since the last call) and clears it. */
q4k_status q4k_last_device_status(void* stream);

/* Test hook for the bounded device-side waits (failure detection without a GPU
 * fault; hipEngine 0.3.0 README, "Core principles": fail closed instead of
 * hanging or falling back). Sets, for every later launch on the current device:
 *   drop_stage     >= 0: the weight producer of every CTA of q4k_gemm and of the
 *                  decode GEMVs skips its stage with this index (no copy, no
 *                  arrival), so the roles waiting for it reach the wait limit;
 *                  < 0: off (the default).
 *   wait_limit_ns  the limit of every bounded wait, in ns; 0 restores the
 *                  default (2 s).
 * A kernel whose wait expires latches Q4K_ERR_DEVICE_TIMEOUT, stops every role,
 * waits (bounded) for its own copies in flight, releases its tensor memory and
 * returns; its outputs are then undefined. Synchronous with the host (a copy to
 * device symbols); not for use while kernels of this library are in flight.
 * Returns Q4K_ERR_CUDA if the copy fails. */
q4k_status q4k_test_wait_fault(int drop_stage, uint64_t wait_limit_ns);

/* Static description of a status code. */
const char* q4k_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* Q4K_H */
