// Shared device helpers and internal launch declarations of libw4a16.
//
// Packed weight layout (see include/w4a16.h): 128-row blocks, 32-code chunks of
// 16 bytes, row-minor inside a chunk column, so one 16-byte load per thread of
// a warp reads 32 consecutive rows' chunks as 512 contiguous bytes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>

#include "../../include/w4a16.h"

namespace w4a16 {

constexpr int kGroup = 128;      // quantisation group along K
constexpr int kRowBlock = 128;   // rows per packed block
constexpr int kChunkK = 32;      // codes per 16-byte chunk

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- loads ----

// 16-byte streaming load through the non-coherent path, no L1 allocation:
// every weight byte is read exactly once per call.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
  uint32_t d;
  // (a & b) | c  ->  immLut = (0xF0 & 0xCC) | 0xAA = 0xEA
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));
  return d;
}

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Per-(row, group) constants of the in-register dequantisation.
struct GroupConsts {
  uint32_t z1024;   // half2(1024 + z, 1024 + z)
  uint32_t zneg64;  // half2(-(64 + z), -(64 + z))
  uint32_t s2;      // half2(s, s)
};

__device__ __forceinline__ GroupConsts make_group_consts(uint32_t z, uint16_t s) {
  GroupConsts c;
  uint32_t a = 0x6400u | z;          // fp16 1024 + z (ulp 1 in [1024, 2048))
  uint32_t b = 0xD400u | (z << 4);   // fp16 -(64 + z) (ulp 1/16 in [64, 128))
  c.z1024 = a | (a << 16);
  c.zneg64 = b | (b << 16);
  c.s2 = (uint32_t)s | ((uint32_t)s << 16);
  return c;
}

// Dequantise the 8 codes of one packed 32-bit word into 4 half2 values
// (k offsets (0,1), (2,3), (4,5), (6,7)), each exactly fp16_RN((q - z) * s):
//  * OR-ing a code into the mantissa of fp16 1024 gives 1024 + q exactly;
//    a code left in bits 4..7 gives 1024 + 16 q exactly;
//  * subtracting 1024 + z, or fma by 1/16 then adding -(64 + z), gives the
//    exact small integer q - z (every intermediate is representable);
//  * one fp16 multiply by s then rounds the exact product once, to nearest
//    even, which is the definition.
__device__ __forceinline__ void dequant_word(uint32_t w, const GroupConsts& c, uint32_t out[4]) {
  const uint32_t kMagic = 0x64006400u;
  const uint32_t kSixteenth = 0x2C002C00u;  // half2(1/16, 1/16)
  uint32_t w8 = w >> 8;
  uint32_t e0 = lop3_and_or(w, 0x000F000Fu, kMagic);
  uint32_t e1 = lop3_and_or(w, 0x00F000F0u, kMagic);
  uint32_t e2 = lop3_and_or(w8, 0x000F000Fu, kMagic);
  uint32_t e3 = lop3_and_or(w8, 0x00F000F0u, kMagic);
  out[0] = h2_mul(h2_sub(e0, c.z1024), c.s2);
  out[1] = h2_mul(h2_fma(e1, kSixteenth, c.zneg64), c.s2);
  out[2] = h2_mul(h2_sub(e2, c.z1024), c.s2);
  out[3] = h2_mul(h2_fma(e3, kSixteenth, c.zneg64), c.s2);
}

// Zero code of row r (0..127) in the 64-byte zero block of one (block, group).
__device__ __forceinline__ uint32_t zero_code(const uint8_t* zblock, int r) {
  return (zblock[r >> 1] >> ((r & 1) * 4)) & 0xFu;
}

// ----------------------------------------------- add + RMS normalisation ----

// The arithmetic of the residual add + RMS normalisation, shared by its own
// kernel and by the decode kernel's normalising prologue so that both give
// the same bits: r = fp16_RN(h + d) pairwise, the sum of squares of r in
// fp32 with one fma per channel in channel order, X = fp16_RN((r * inv) * g).
__device__ __forceinline__ uint32_t hadd2_rn(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float lo_f(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
}

__device__ __forceinline__ float hi_f(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}

__device__ __forceinline__ float sum_sq2(uint32_t w, float ss) {
  const float a = lo_f(w), b = hi_f(w);
  return fmaf(b, b, fmaf(a, a, ss));
}

// Two channels of X from two of r and two of gamma.
__device__ __forceinline__ uint32_t scale2(uint32_t r, uint32_t g, float inv) {
  const float x0 = __fmul_rn(__fmul_rn(lo_f(r), inv), lo_f(g));
  const float x1 = __fmul_rn(__fmul_rn(hi_f(r), inv), hi_f(g));
  return (uint32_t)__half_as_ushort(__float2half_rn(x0)) |
         ((uint32_t)__half_as_ushort(__float2half_rn(x1)) << 16);
}

// 1 / sqrt(mean + eps) from the fixed-order sum of squares of a row.
__device__ __forceinline__ float rms_inv(float sum_sq, int K, float eps) {
  return __frsqrt_rn(__fadd_rn(__fdiv_rn(sum_sq, (float)K), eps));
}

// Threads per row and 16-byte chunks in flight per thread of the sum of
// squares (its order depends on both).
constexpr int kNormThreads = 256;
constexpr int kNormBatch = 4;

// Inputs of the decode kernel's normalising prologue (h null: none; the
// kernel then reads X).  r_out may be null.
struct NormIn {
  const uint16_t* h;
  const uint16_t* d;
  const uint16_t* gamma;
  float eps;
  uint16_t* r_out;
};

// ------------------------------------------------------ gate/up rows ----

// The gate/up row order of w4a16_pack_gate_up: packed block b holds the 64
// intermediate channels i = 64 b + 16 q + j (q = 0..3 the 32-row lane quarter,
// j = 0..15), the gate row of channel i at packed row 32 q + j and its up row
// at 32 q + 16 + j, so one warp of an epilogue (thread = packed row) holds
// both halves of 16 channels and pairs them with one shuffle.
__host__ __device__ inline int gate_up_channel(int b, int r) { return b * 64 + (r >> 5) * 16 + (r & 15); }

// Canonical row held by packed row r of block b (-1: a padding row).  mi == 0:
// rows in order, M of them; mi > 0: the gate/up order over a canonical weight
// whose rows are the gate projection's mi rows then the up projection's mi.
__host__ __device__ inline int packed_source_row(int b, int r, int M, int mi) {
  if (mi == 0) {
    const int m = b * kRowBlock + r;
    return m < M ? m : -1;
  }
  const int i = gate_up_channel(b, r);
  if (i >= mi) return -1;
  return (r & 16) ? mi + i : i;
}

// --------------------------------------------------------- output map ----

// Epilogue kinds of the GEMM kernels.
enum Epi : int {
  kEpiPlain = 0,    // Y[n][m], one RNE rounding of the fp32 accumulator
  kEpiQkv = 1,      // three outputs plus an optional bias (w4a16_gemm_qkv)
  kEpiGateUp = 2,   // H[n][i] = silu(gate) * up (w4a16_gemm_gate_up)
};

// Where an epilogue puts row m of the result when the caller asked for a
// fused form.  QKV (w4a16_gemm_qkv): rows [0, end0), [end0, end1) and
// [end1, M) go to three token-major outputs of their own widths, each value
// after adding an optional fp16 bias of its row in fp32 and one RNE rounding
// to fp16.  Gate/up (w4a16_gemm_gate_up): h [N][mi], from a weight packed in
// the gate/up row order.
struct OutMap {
  int kind;               // Epi: kEpiQkv or kEpiGateUp
  uint16_t* y0;
  uint16_t* y1;
  uint16_t* y2;
  int end0, end1;
  const uint16_t* bias;   // [M] or null
  uint16_t* h;
  int mi;
};

// Row m's destination in the fused form, resolved once per row: its element
// in token 0 of the output it belongs to, that output's row pitch (its
// width) and the fp32 value of its bias (0 when there is none).
struct RowDst {
  uint16_t* y;
  int ld;
  float bias;
};

__device__ __forceinline__ RowDst row_dst(const OutMap& o, int M, int m) {
  RowDst d;
  if (m < o.end0) {
    d.y = o.y0 + m;
    d.ld = o.end0;
  } else if (m < o.end1) {
    d.y = o.y1 + (m - o.end0);
    d.ld = o.end1 - o.end0;
  } else {
    d.y = o.y2 + (m - o.end1);
    d.ld = M - o.end1;
  }
  d.bias = o.bias ? __half2float(__ushort_as_half(o.bias[m])) : 0.0f;
  return d;
}

// Token n of row d: the accumulator plus the bias in fp32 (skipped without a
// bias, so a zero result keeps its sign), rounded once to fp16.
__device__ __forceinline__ void store_row(const RowDst& d, bool has_bias, int n, float v) {
  if (has_bias) v = __fadd_rn(v, d.bias);
  d.y[(size_t)n * d.ld] = __half_as_ushort(__float2half_rn(v));
}

// Gate/up epilogue of one token: v is the fp32 accumulator of packed row r
// (0..127, thread = row, all 32 lanes of the warp calling together) of block
// b.  Lanes 0..15 hold gate rows and take their channel's up value from lane
// + 16, then write H[n][i] = fp16_RN(silu(g) * u), silu(g) = g / (1 + e^-g),
// in fp32 with the hardware exponential and approximate division (a few fp32
// ulps, far below the one fp16 rounding of H; e^-g overflowing to infinity
// gives silu = -0, not NaN; the accurate forms cost the tile kernel 8 % more
// at LLaMA-7B gate/up, N = 4096).  The decode kernels call this per token;
// the tile kernel pairs tokens with the same arithmetic in its epilogue.
__device__ __forceinline__ void store_gate_up(const OutMap& o, int b, int r, int n, float v, bool valid) {
  const float u = __shfl_down_sync(0xffffffffu, v, 16);
  const int i = gate_up_channel(b, r);
  if (valid && (r & 16) == 0 && i < o.mi) {
    const float silu = __fdividef(v, 1.0f + __expf(-v));
    o.h[(size_t)n * o.mi + i] = __half_as_ushort(__float2half_rn(silu * u));
  }
}

// ------------------------------------------------------- launch helpers ----

// SM count of the current device (cached per device; 148 if it cannot be read).
int num_sms();

// Tensor map of X [N][K] fp16 for the tensor-core kernels: boxes of 64 k x
// box_rows tokens x `slabs` 64-k slabs, 128-byte swizzle, zero fill past N.
cudaError_t make_x_map(CUtensorMap* map, const uint16_t* X, int N, int K, int box_rows, int slabs);

// Raise a kernel's dynamic shared-memory limit on the current device, once
// per device (bit `dev` of `done`).  Two threads racing on the first call
// both set the same value, which is harmless.
inline cudaError_t ensure_smem_limit(const void* fn, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// GEMV (CUDA cores): N in 1..kGemvMaxTokens per launch.
constexpr int kGemvMaxTokens = 8;
// Tokens of one plain / QKV / gate-up launch: 9 to 16 run as two 8-token
// MMA column blocks sharing the dequantised weights (the normalising
// prologue keeps kGemvMaxTokens).
constexpr int kGemvWideTokens = 16;

// om: null for the plain [N][M] output Y, else the fused output map (Y unused).
// With pdl the launch may overlap the previous kernel in the stream: the
// first weight stages are read before the grid dependency wait, X and Y
// after it.
// norm: the normalising prologue (X unused; N <= kGemvMaxTokens).
cudaError_t launch_gemv(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                        const uint16_t* X, uint16_t* Y, int M, int K, int N,
                        cudaStream_t stream, const OutMap* om = nullptr, bool pdl = false,
                        const NormIn* norm = nullptr);

// Residual add + RMS normalisation: one CTA per token row, K a multiple of 8
// and at most kMaxNormK (the row's residual is held in shared memory).
constexpr int kMaxNormK = 1 << 16;
cudaError_t launch_add_rmsnorm(const uint16_t* h, const uint16_t* d, const uint16_t* gamma, float eps,
                               int N, int K, uint16_t* r_out, uint16_t* X, cudaStream_t stream);

cudaError_t launch_quantize(const uint16_t* W, int M, int K, uint8_t* q, uint16_t* scales, uint8_t* zeros,
                            cudaStream_t stream);

// mi > 0: the gate/up row order (packed_source_row), M = 2 mi.
cudaError_t launch_pack(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                        int M, int K, uint8_t* wq_p, uint16_t* s_p, uint8_t* z_p,
                        cudaStream_t stream, int mi = 0);

cudaError_t launch_dequant(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           uint16_t* W, int M, int K, cudaStream_t stream);

// Tensor-core path.  Returns cudaErrorNotSupported when the sizes are outside
// what the kernel handles.
cudaError_t launch_gemm_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           const uint16_t* X, uint16_t* Y, int M, int K, int N,
                           cudaStream_t stream, const OutMap* om = nullptr);

// Decode GEMV / few-token product on the tensor cores, split along the
// weight stream over every SM (N in 1..kGemvTcMaxTokens).  The caller's
// workspace holds one counter per (row block, lane quarter), zero between
// calls, then the fp32 partials of the blocks split between CTAs.  With pdl
// the launch may overlap the previous kernel in the stream: the weights are
// read before the grid dependency wait, X, Y and the workspace after it.
constexpr int kGemvTcMaxTokens = 64;
size_t gemv_tc_counter_bytes(int M);
// w4a16_gemm_noalloc: the same kernel on a fixed device array of this many
// bytes instead of a caller workspace (cudaErrorNotSupported when the sizes
// need more).
constexpr size_t kNoallocScratchBytes = (size_t)4 << 20;
cudaError_t launch_gemv_tc_noalloc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                                   const uint16_t* X, uint16_t* Y, int M, int K, int N, bool pdl,
                                   cudaStream_t stream);
size_t gemv_tc_workspace_bytes(int M, int K, int N);
cudaError_t launch_gemv_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros, const uint16_t* X,
                           uint16_t* Y, int M, int K, int N, void* workspace, bool pdl, cudaStream_t stream,
                           const OutMap* om = nullptr);

// Read-and-clear of the per-kernel-family device status words (1 = a bounded
// wait ran out).
cudaError_t read_and_clear_tc_status(int* v);
cudaError_t read_and_clear_gemv_status(int* v);
cudaError_t read_and_clear_gvtc_status(int* v);

// Diagnostic: a kernel whose bounded wait must run out (see
// w4a16_selftest_wait_timeout).
cudaError_t launch_wait_timeout_selftest(long long limit_cycles, cudaStream_t stream);

}  // namespace w4a16
