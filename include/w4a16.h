/*
 * w4a16.h -- C ABI of the B200 (sm_100a) W4A16 group-128 linear layer.
 *
 * The operation ("PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1, GEMM
 * definition; item 2, GEMV as its n = 1 case; section 3.1, AWQ weight-only
 * int4 quantisation with group_size 128 and a scale and a zero per group):
 *
 *     Y[n][m] = sum_k  w[m][k] * X[n][k],     w[m][k] = fp16_RN((q[m][k] - z[m][g]) * s[m][g]),
 *     g = k / 128,  q, z in 0..15 (unsigned 4-bit),  s fp16,  X, Y fp16,
 *
 * i.e. Y = X . dequant(W)^T with X token-major [N][K] and Y token-major [N][M]
 * (the same memory as column-major X[K][N] and Y[M][N]).  The products are
 * accumulated in fp32 and Y is rounded once to fp16 (round to nearest even).
 *
 * Conventions for every entry point
 *   - Buffers are owned by the caller.  The library allocates no device
 *     memory and never synchronises the stream it is given.
 *   - Pointers named "device" must be device (or managed) memory of the
 *     current CUDA device; every one must be 16-byte aligned.
 *   - Argument checks run on the host before any launch and return an error
 *     code without touching the GPU.  Launch failures are reported as
 *     W4A16_ERR_CUDA.  Nothing is thrown and nothing exits.
 *   - An output buffer may not share a byte with an input or with another
 *     output of the same call (W4A16_ERR_INVALID_ARG), except where a call
 *     allows in-place use (the residual of w4a16_add_rmsnorm).
 *   - Calls are asynchronous on `stream` (0 = the legacy default stream).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W4A16_API __attribute__((visibility("default")))
#else
#define W4A16_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A16_OK = 0,
    W4A16_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad path */
    W4A16_ERR_UNSUPPORTED = 2,  /* group != 128, K % 128 != 0, sizes too big */
    W4A16_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
    W4A16_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    W4A16_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out */
    W4A16_ERR_BOUNDS = 6        /* libw4a16_debug.so only (built with -DW4A16_DEBUG_BOUNDS):
                                   an in-kernel index check of the decode kernel found an
                                   access outside its buffer; the access was skipped */
} w4a16_status;

/* Kernel selection for w4a16_gemm_ex and w4a16_gemm_ws. */
typedef enum {
    W4A16_PATH_AUTO = 0,     /* choose by N and M: GEMV for N <= 8, and for N <= 16
                                when M <= 8192; TC above */
    W4A16_PATH_GEMV = 1,     /* decode kernel: weights streamed to registers, warp-level
                                MMAs (any N; 8 tokens per launch, 16 when M <= 4096) */
    W4A16_PATH_TC = 2,       /* tcgen05 tile kernel (any N) */
    W4A16_PATH_GEMV_TC = 3   /* tcgen05 decode kernel, weight stream split over every SM
                                (N <= 64; needs a workspace; never chosen by AUTO: slower
                                than GEMV and TC at every N measured) */
} w4a16_path;

/*
 * The residual add + RMS normalisation fused into the QKV projection's
 * prologue ("PerfXLLM on Snapdragon 8 Gen2", section 3.2: the residual
 * addition and the normalisation are fused so their result does not go
 * through global memory; here that result, X, is formed inside the
 * projection itself and never stored).  For N <= 8 tokens, one launch of the
 * decode kernel computes
 *     r = fp16_RN(h + d)                      (d NULL: r = h)
 *     X = fp16_RN((r * inv) * gamma),  inv = 1 / sqrt(mean(r^2) + eps)
 * exactly as w4a16_add_rmsnorm (the same bits), then the outputs of
 * w4a16_gemm_qkv from that X, and writes r to r_out when r_out is not NULL.
 *   h, d, r_out  device fp16 [N][K], 16-byte aligned; r_out must not overlap
 *                h or d (no in-place update here) nor any other argument.
 *   gamma        device fp16 [K], 16-byte aligned; eps >= 0.
 *   flags        0 or W4A16_FLAG_EARLY_WEIGHTS (the weights are read before
 *                the previous kernel completes, h and d after it).
 *   weight, bias, Mq, Mk, Mv, outputs: as w4a16_gemm_qkv.
 * W4A16_ERR_UNSUPPORTED for N > 8 (run w4a16_add_rmsnorm, then
 * w4a16_gemm_qkv); other errors as w4a16_gemm_qkv and w4a16_add_rmsnorm.
 */
W4A16_API w4a16_status w4a16_add_rmsnorm_gemm_qkv(const uint16_t* h, const uint16_t* d,
                           const uint16_t* gamma, float eps, uint16_t* r_out,
                           const void* wq_packed, const void* scales_packed,
                           const void* zeros_packed, const uint16_t* bias,
                           int Mq, int Mk, int Mv, int K, int N, int group,
                           uint16_t* Yq, uint16_t* Yk, uint16_t* Yv,
                           unsigned flags, void* stream);

/* Flags of the workspace entry points (w4a16_gemm_ws, w4a16_gemm_qkv_ws,
 * w4a16_gemm_gate_up_ws). */
#define W4A16_FLAG_EARLY_WEIGHTS 1u
/*   On the decode paths (W4A16_PATH_GEMV, W4A16_PATH_GEMV_TC), launch with
 *   programmatic dependent launch: the call's CTAs may start, and read the
 *   packed weight, while the previous kernel in the stream is still running;
 *   X, the bias, Y and the workspace are only touched after that kernel has
 *   completed.  The caller guarantees that no kernel still running writes the
 *   packed weight (true of weights loaded once, before inference).  Ignored
 *   by the tensor-core tile path. */

/* Human-readable name of a status code.  Never returns NULL. */
W4A16_API const char* w4a16_status_string(int status);

/*
 * Packed-weight sizes, in bytes, for an M x K weight with the given group.
 * "PerfXLLM on Snapdragon 8 Gen2", section 3.1: int4 codes take a quarter of
 * the fp16 weight and the scale and zero of each group of 128 about 1 % more;
 * the layout below is this library's own (section 3.3 asks for vectorised
 * weight loads, which the 16-byte row-interleaved chunks serve).
 *
 * Packed layout (all three buffers are padded to Mp = ceil(M / 128) * 128 rows;
 * padding rows hold q = 0, z = 0, s = 0, i.e. zero weights):
 *   wq     : Mp * K / 2 bytes.  16-byte chunk (b, c, r) at byte offset
 *            ((b * K/32 + c) * 128 + r) * 16 holds the 32 codes
 *            q[128 b + r][32 c + j], j = 0..31, as four little-endian 32-bit
 *            words; word j/8 keeps the 8 codes of j = 8t..8t+7 with the code of
 *            offset o = j % 8 in nibble p = o/2 (o even) or 4 + o/2 (o odd),
 *            nibble p occupying bits 4p..4p+3.  A row's codes for offsets
 *            (2i, 2i+1) thus sit 16 bits apart, which lets one mask-and-or
 *            form both as fp16 values 1024 + q.
 *   scales : Mp * K/128 * 2 bytes, fp16 at ((b * K/128 + g) * 128 + r).
 *   zeros  : Mp * K/128 / 2 bytes, byte ((b * K/128 + g) * 64 + r/2), low
 *            nibble for even r, high nibble for odd r.
 * Metadata is 2.5 bytes per group of 128 weights (about 1 % of the fp16
 * weight size, 3.9 % of the int4 size).
 *
 * Returns W4A16_ERR_INVALID_ARG for null outputs or M, K <= 0,
 * W4A16_ERR_UNSUPPORTED for group != 128 or K % 128 != 0.
 */
W4A16_API w4a16_status w4a16_packed_sizes(int M, int K, int group,
                                size_t* wq_bytes, size_t* scales_bytes,
                                size_t* zeros_bytes);

/*
 * Group quantiser: fp16 W -> canonical (q, scales, zeros), the step before
 * w4a16_pack (offline).  "PerfXLLM on Snapdragon 8 Gen2", section 3.1 fixes
 * 4-bit codes, groups of 128 along K and one scale and one zero per group;
 * the rounding rule is min-max asymmetric with 0 inside the range, every step
 * an IEEE fp32 operation (round to nearest even), per (row, group):
 *     lo = min(0, min w), hi = max(0, max w), r = max(hi - lo, 2^-14),
 *     s = fp16_RN(r / 15), f = 1 / s, z = clamp(rint(-lo f), 0, 15),
 *     q = clamp(rint(w f) + z, 0, 15).
 *   W       device fp16  [M][K], 16-byte aligned, finite values
 *   q       device uint8 [M][K], 16-byte aligned (output)
 *   scales  device fp16  [M][K/128], 2-byte aligned (output)
 *   zeros   device uint8 [M][K/128] (output)
 * W4A16_ERR_UNSUPPORTED for group != 128 or K % 128 != 0.
 */
W4A16_API w4a16_status w4a16_quantize(const uint16_t* W, int M, int K, int group,
                            uint8_t* q, uint16_t* scales, uint8_t* zeros, void* stream);

/*
 * Residual add + RMS normalisation: the operator that produces X for the
 * projections.  "PerfXLLM on Snapdragon 8 Gen2", section 3.2, first fusion:
 * the residual connection's addition and the normalisation are one operator,
 * so their intermediate does not travel through global memory.  Per token row
 * n (reading of the page, which names the two operations only):
 *     r[n][k] = fp16_RN(h[n][k] + d[n][k])                 (d == NULL: r = h)
 *     X[n][k] = fp16_RN((r[n][k] * inv) * gamma[k]),  inv = 1 / sqrt(eps + (1/K) sum_k r[n][k]^2)
 * with the mean, the root and the products in fp32 and one rounding of X.
 *   h      device fp16 [N][K], the residual stream
 *   d      device fp16 [N][K] added to it, or NULL
 *   gamma  device fp16 [K], the normalisation weight
 *   eps    finite, >= 0
 *   r_out  device fp16 [N][K], the new residual, or NULL not to write it; may be
 *          h or d itself (updated in place), must not partly overlap either
 *   X      device fp16 [N][K]; must not overlap h, d, gamma or r_out
 * Every pointer 16-byte aligned; N >= 1; K a multiple of 8, at most 65536.
 * W4A16_ERR_INVALID_ARG for null h, gamma or X, N or K <= 0, a negative or
 * non-finite eps, or overlapping buffers; W4A16_ERR_UNSUPPORTED for K % 8 != 0
 * or K > 65536.
 */
W4A16_API w4a16_status w4a16_add_rmsnorm(const uint16_t* h, const uint16_t* d, const uint16_t* gamma,
                               float eps, int N, int K, uint16_t* r_out, uint16_t* X, void* stream);

/*
 * Canonical -> packed layout (offline; not on the per-token path).
 * "PerfXLLM on Snapdragon 8 Gen2", section 3.1 (int4 codes, group 128, a
 * scale and a zero per group) and section 3.3 (vectorised weight access).
 * Argument order: codes, then the fp16 scales, then the zeros (the order of
 * the packed buffers w4a16_packed_sizes reports).
 *   q       device uint8  [M][K], values 0..15 (higher bits are ignored)
 *   scales  device fp16   [M][K/128]
 *   zeros   device uint8  [M][K/128], values 0..15 (higher bits are ignored)
 *   wq_packed, scales_packed, zeros_packed: device outputs of the sizes
 *   w4a16_packed_sizes returns.  Inputs need only natural alignment; the
 *   outputs must be 16-byte aligned.
 */
W4A16_API w4a16_status w4a16_pack(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                        int M, int K, int group,
                        void* wq_packed, void* scales_packed, void* zeros_packed,
                        void* stream);

/*
 * The gate/up row order, for w4a16_gemm_gate_up: canonical -> packed like
 * w4a16_pack, for a weight of 2 * Mi rows whose rows [0, Mi) are the gate
 * projection and rows [Mi, 2 Mi) the up projection (q [2 Mi][K], scales and
 * zeros [2 Mi][K/128], as w4a16_pack).  Packed block b (128 rows) holds the
 * intermediate channels i = 64 b + 16 q + j (q = 0..3, j = 0..15): the gate
 * row of channel i as packed row 32 q + j, its up row as packed row
 * 32 q + 16 + j; rows of channels i >= Mi are zero.  Output sizes are those
 * of w4a16_packed_sizes(2 * Mi, K, group).  Errors as w4a16_pack, plus
 * W4A16_ERR_INVALID_ARG for Mi <= 0.
 */
W4A16_API w4a16_status w4a16_pack_gate_up(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                                int Mi, int K, int group,
                                void* wq_packed, void* scales_packed, void* zeros_packed,
                                void* stream);

/*
 * The gate/up projection with its activation fused into the epilogue
 * ("PerfXLLM on Snapdragon 8 Gen2", section 3.2: operator fusion removes an
 * intermediate's write to and read from global memory; the page lists the
 * add + normalisation, merged-QKV and attention fusions, and this extends the
 * principle to the feed-forward block).  With g and u the fp32 accumulators
 * of channel i's gate and up rows (as w4a16_gemm computes them):
 *     H[n][i] = fp16_RN(silu(g) * u),   silu(g) = g / (1 + e^(-g)),
 * in fp32, one rounding to fp16; the [N][2 Mi] product is never written.
 *   wq_packed, scales_packed, zeros_packed: packed by w4a16_pack_gate_up
 *   X  device fp16 [N][K];  H  device fp16 [N][Mi] (token-major), written in full.
 * Kernel choice as w4a16_gemm for M = 2 Mi; errors as w4a16_gemm, plus
 * W4A16_ERR_INVALID_ARG for Mi <= 0.
 */
W4A16_API w4a16_status w4a16_gemm_gate_up(const void* wq_packed, const void* scales_packed,
                                const void* zeros_packed, const uint16_t* X, uint16_t* H,
                                int Mi, int K, int N, int group, void* stream);

/* w4a16_gemm_gate_up with a forced path (w4a16_path) and the workspace and
 * flags of w4a16_gemm_ws (workspace size: w4a16_gemm_workspace_size(2 Mi, K,
 * N, group)). */
W4A16_API w4a16_status w4a16_gemm_gate_up_ws(const void* wq_packed, const void* scales_packed,
                                   const void* zeros_packed, const uint16_t* X, uint16_t* H,
                                   int Mi, int K, int N, int group, int path,
                                   void* workspace, size_t workspace_bytes, unsigned flags, void* stream);

/*
 * Y[N][M] = X[N][K] . dequant(W)[M][K]^T   (fp16 in, fp32 accumulate, fp16 out)
 * "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1 (C[m, n] = A[m, k]
 * B[k, n]) and item 2 (the GEMV is its n = 1 case); the weight is the
 * section 3.1 int4 group-128 format.
 *   wq_packed, scales_packed, zeros_packed: device, packed as above.
 *   X  device fp16 [N][K] (token-major), 16-byte aligned.
 *   Y  device fp16 [N][M] (token-major), 16-byte aligned; fully overwritten.
 *   M >= 1, N >= 1, K a positive multiple of 128, group == 128.
 * The result is deterministic: the same inputs give the same bits.
 */
W4A16_API w4a16_status w4a16_gemm(const void* wq_packed, const void* scales_packed,
                        const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                        int M, int K, int N, int group, void* stream);

/*
 * The fused-projection form ("PerfXLLM on Snapdragon 8 Gen2", section 3.2:
 * operator fusion removes intermediate reads and writes, and the three
 * matrix products that make Q, K and V become one larger product).  The
 * weight's rows are three projections stacked, M = Mq + Mk + Mv; the result
 * goes straight to three token-major outputs instead of one [N][M] buffer:
 *     Yq[n][m]      = fp16_RN(acc[n][m]           + bias[m])           m < Mq
 *     Yk[n][m]      = fp16_RN(acc[n][Mq + m]      + bias[Mq + m])      m < Mk
 *     Yv[n][m]      = fp16_RN(acc[n][Mq + Mk + m] + bias[Mq + Mk + m]) m < Mv
 * with acc the fp32 accumulator of w4a16_gemm and the bias added in fp32
 * (bias device fp16 [M], 2-byte aligned, or NULL for none).  Mq, Mk, Mv >= 1; other
 * arguments, alignment (Yq, Yk, Yv 16-byte aligned) and kernel choice as
 * w4a16_gemm.
 */
W4A16_API w4a16_status w4a16_gemm_qkv(const void* wq_packed, const void* scales_packed,
                            const void* zeros_packed, const uint16_t* X, const uint16_t* bias,
                            int Mq, int Mk, int Mv, int K, int N, int group,
                            uint16_t* Yq, uint16_t* Yk, uint16_t* Yv, void* stream);

/*
 * Workspace of w4a16_gemm_ws / w4a16_gemm_qkv_ws / w4a16_gemm_gate_up_ws
 * for an M x K weight and N tokens on the current device (it depends on the
 * device's SM count), in bytes: enough for the automatic choice and for a
 * forced W4A16_PATH_GEMV_TC; 0 for N > 64, where no path needs one.  The size
 * grows with N, so a workspace sized for the largest N serves every smaller
 * one.  W4A16_ERR_INVALID_ARG / W4A16_ERR_UNSUPPORTED as w4a16_gemm.
 */
W4A16_API w4a16_status w4a16_gemm_workspace_size(int M, int K, int N, int group, size_t* bytes);

/*
 * w4a16_gemm with a caller-owned workspace, which lets the decode and
 * few-token product run on every SM ("PerfXLLM on Snapdragon 8 Gen2",
 * section 3.3 item 2: the GEMV is memory bound; the weight is tiled along
 * both its rows and K so the whole device streams it).  With path AUTO it
 * chooses as w4a16_gemm; forced W4A16_PATH_GEMV_TC (N <= 64): CTA c of G streams units
 * [c U / G, (c + 1) U / G) of the U = ceil(M/128) * K/128 (row block, group)
 * units; a block split between CTAs is summed, in CTA order, from fp32
 * partials in the workspace, so the result stays deterministic.
 *   workspace  device, 16-byte aligned, at least w4a16_gemm_workspace_size
 *              bytes; its contents on entry do not matter: each call on the
 *              split path first clears the counters it uses (an asynchronous
 *              memset on `stream`), and a completed call leaves them at zero.
 *              One workspace serves any number of calls in one stream; calls
 *              that may run at the same time (different streams) need
 *              different workspaces.
 *   workspace_bytes  its size.
 *   flags      0 or W4A16_FLAG_EARLY_WEIGHTS.
 * W4A16_ERR_INVALID_ARG when the forced path needs a workspace that is
 * missing or too small, or when the workspace overlaps another buffer; other
 * arguments as w4a16_gemm_ex.  workspace may be NULL (workspace_bytes 0):
 * AUTO then chooses as w4a16_gemm.
 */
W4A16_API w4a16_status w4a16_gemm_ws(const void* wq_packed, const void* scales_packed,
                           const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                           int M, int K, int N, int group, int path,
                           void* workspace, size_t workspace_bytes, unsigned flags, void* stream);

/* w4a16_gemm_qkv with a workspace: the fused QKV form on the kernel
 * w4a16_gemm_ws would choose for M = Mq + Mk + Mv (automatic choice only);
 * workspace and flags as there. */
W4A16_API w4a16_status w4a16_gemm_qkv_ws(const void* wq_packed, const void* scales_packed,
                               const void* zeros_packed, const uint16_t* X, const uint16_t* bias,
                               int Mq, int Mk, int Mv, int K, int N, int group,
                               uint16_t* Yq, uint16_t* Yk, uint16_t* Yv,
                               void* workspace, size_t workspace_bytes, unsigned flags, void* stream);

/* As w4a16_gemm, with the kernel forced (w4a16_path).  W4A16_PATH_AUTO is the
 * same as w4a16_gemm.  Used by tests and the benchmark to time the kernels
 * side by side ("PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1: each
 * regime, few tokens or many, gets its own tiling).  W4A16_PATH_GEMV_TC needs
 * a workspace, so it is W4A16_ERR_INVALID_ARG here (use w4a16_gemm_ws). */
W4A16_API w4a16_status w4a16_gemm_ex(const void* wq_packed, const void* scales_packed,
                           const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                           int M, int K, int N, int group, int path, void* stream);

/* The path w4a16_gemm would take for these sizes (a w4a16_path value other
 * than AUTO), or -1 if the sizes are invalid.  Host only; touches no GPU.
 * "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1: the operator switches
 * tiling with the number of tokens; the crossovers here are measured. */
W4A16_API int w4a16_select_path(int M, int K, int N);

/*
 * w4a16_gemm on the split decode kernel (W4A16_PATH_GEMV_TC) without any
 * allocation, for callers that cannot call cudaMalloc: plug-ins inside a
 * framework whose caching allocator or fixed arena owns all device memory
 * (a cudaMalloc behind its back fragments or overcommits it), and servers
 * that reserve their whole memory budget at start-up and may not allocate
 * afterwards.  Such callers also have no workspace to hand to
 * w4a16_gemm_ws.  The papers have no counterpart to this entry point: it is
 * an interface choice of this library.
 *   The kernel's scratch (split-block counters and fp32 partials) is a
 *   file-scope device array of 4 MiB, held by every GPU that loads the
 *   library until the process exits.  Sizes whose scratch
 *   (w4a16_gemm_workspace_size) exceeds 4 MiB, or N > 64, return
 *   W4A16_ERR_UNSUPPORTED; on a 148-SM device that allows N <= 16 for every
 *   LLaMA shape.
 *   The first call on a device looks up the array's address with that device
 *   current (cudaGetSymbolAddress); make that first call before any stream
 *   capture.  Each call clears the counters (an asynchronous memset on
 *   `stream`) and then launches the kernel.
 *   Every call on a device shares the one array, which keeps the last call's
 *   contents: calls that overlap on the GPU (different streams, or
 *   programmatic overlap with another such call) race on it and must be
 *   ordered by the caller.
 *   flags as w4a16_gemm_ws; other arguments as w4a16_gemm_ex.
 */
W4A16_API w4a16_status w4a16_gemm_noalloc(const void* wq_packed, const void* scales_packed,
                           const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                           int M, int K, int N, int group, unsigned flags, void* stream);

/* The path w4a16_gemm_ws with a workspace would take. */
W4A16_API int w4a16_select_path_ws(int M, int K, int N);

/*
 * Writes the dequantised weight W[m][k] = fp16_RN((q - z) * s) as fp16,
 * row-major [M][K], from the packed buffers ("PerfXLLM on Snapdragon 8 Gen2",
 * section 3.1: int4 with a scale and a zero per group of 128; the formula and
 * its single rounding are this library's reading of that passage).  The values are bit-identical to
 * what the GEMM kernels multiply; parity checks compare them with an
 * independent CPU computation.
 */
W4A16_API w4a16_status w4a16_dequant_debug(const void* wq_packed, const void* scales_packed,
                                 const void* zeros_packed, uint16_t* W_out,
                                 int M, int K, int group, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device-side status words
 * that bounded waits inside the kernels set when they give up.
 * Writes W4A16_OK, W4A16_ERR_TIMEOUT or (debug build) W4A16_ERR_BOUNDS to
 * *status.  Not for the hot path.
 * The words are per device, shared by every stream, and read and cleared by
 * two separate copies: the answer is exact only while no other stream runs
 * this library's kernels on the device (a timeout recorded between the two
 * copies would be cleared unseen).
 */
W4A16_API w4a16_status w4a16_device_status(void* stream, int* status);

/*
 * Diagnostic for the failure-detection path: launches one tiny kernel that
 * waits on an mbarrier nothing ever completes, with a budget of limit_cycles
 * SM clock cycles (0 .. 2^32).  The wait gives up, records a timeout in the
 * device status word and the kernel returns normally, so the next
 * w4a16_device_status reports W4A16_ERR_TIMEOUT and the CUDA context stays
 * usable.  Returns W4A16_ERR_INVALID_ARG for a limit outside that range.
 */
W4A16_API w4a16_status w4a16_selftest_wait_timeout(long long limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
