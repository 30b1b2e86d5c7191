// On-device group quantiser fp16 W -> (q, s, z), the step before w4a16_pack.
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.1: the weights alone are
// quantised, to 4-bit integers, in groups of 128 along K with one scale and
// one zero per group.  The page gives no rounding rule; the one used here is
// min-max asymmetric with 0 inside the range, every decision an IEEE fp32
// operation rounded to nearest even (so any implementation taking the same
// fp32 steps gets the same codes):
//
//   lo = min(0, min w), hi = max(0, max w); r = hi - lo, at least 2^-14;
//   s = fp16_RN(r / 15); f = 1 / s; z = clamp(rint(-lo f), 0, 15);
//   q = clamp(rint(w f) + z, 0, 15).
//
// A half-warp per (row, group): lane l of the half reads the group's weights
// 8l .. 8l + 7 (16 bytes; the half reads the group's 256 contiguous bytes).
// A warp takes 8 groups and issues all its loads before any arithmetic, so
// 64 bytes per lane are in flight; the minimum and maximum come from
// shuffles within the half-warp, and each lane writes its eight codes as one
// 8-byte store.  Bound by HBM: 2 bytes read and 1 byte written per weight.
#include "w4a16_internal.cuh"

namespace w4a16 {

namespace {

constexpr int kQWarpsPerBlock = 8;
constexpr int kQGroupsPerWarp = 8;                  // two per round, four rounds
constexpr int kQRounds = kQGroupsPerWarp / 2;

__device__ __forceinline__ float fp16_bits_to_float(uint32_t bits) {
  return __half2float(__ushort_as_half((unsigned short)(bits & 0xFFFFu)));
}

__global__ void __launch_bounds__(kQWarpsPerBlock * 32)
quantize_kernel(const uint16_t* __restrict__ W, int M, int K, uint8_t* __restrict__ q,
                uint16_t* __restrict__ s_out, uint8_t* __restrict__ z_out) {
  const int kg = K / kGroup;
  const long long units = (long long)M * kg;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  const long long unit0 =
      ((long long)blockIdx.x * kQWarpsPerBlock + (threadIdx.x >> 5)) * kQGroupsPerWarp + half;

  uint4 raw[kQRounds];
  size_t base[kQRounds];
#pragma unroll
  for (int j = 0; j < kQRounds; ++j) {
    const long long unit = unit0 + 2 * j;
    raw[j] = make_uint4(0, 0, 0, 0);
    base[j] = 0;
    if (unit < units) {
      const int m = (int)(unit / kg);
      const int g = (int)(unit - (long long)m * kg);
      base[j] = (size_t)m * K + (size_t)g * kGroup + 8 * hl;
      raw[j] = __ldg(reinterpret_cast<const uint4*>(W + base[j]));
    }
  }

#pragma unroll
  for (int j = 0; j < kQRounds; ++j) {
    const long long unit = unit0 + 2 * j;
    const uint32_t words[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = fp16_bits_to_float(words[i]);
      v[2 * i + 1] = fp16_bits_to_float(words[i] >> 16);
    }
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo = fminf(lo, v[i]);
      hi = fmaxf(hi, v[i]);
    }
    // Offsets below 16 keep each half-warp (one group) to itself.
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    float r = __fsub_rn(hi, lo);
    const float r_min = 6.103515625e-05f;           // 2^-14
    if (!(r >= r_min)) r = r_min;
    const __half s16 = __float2half_rn(__fdiv_rn(r, 15.0f));
    const float f = __fdiv_rn(1.0f, __half2float(s16));
    const float zf = fminf(fmaxf(rintf(__fmul_rn(-lo, f)), 0.0f), 15.0f);
    uint32_t codes[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float qf = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(v[i], f)), zf), 0.0f), 15.0f);
      codes[i >> 2] |= (uint32_t)qf << (8 * (i & 3));
    }
    if (unit < units) {
      *reinterpret_cast<uint2*>(q + base[j]) = make_uint2(codes[0], codes[1]);
      if (hl == 0) {
        const size_t sz = (size_t)(base[j] / kGroup);   // = m * kg + g
        s_out[sz] = __half_as_ushort(s16);
        z_out[sz] = (uint8_t)zf;
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int M, int K, uint8_t* q, uint16_t* scales, uint8_t* zeros,
                            cudaStream_t stream) {
  const long long units = (long long)M * (K / kGroup);
  const long long per_block = (long long)kQWarpsPerBlock * kQGroupsPerWarp;
  const long long blocks = (units + per_block - 1) / per_block;
  if (blocks > 0x7fffffffLL) return cudaErrorNotSupported;
  quantize_kernel<<<(unsigned)blocks, kQWarpsPerBlock * 32, 0, stream>>>(W, M, K, q, scales, zeros);
  return cudaGetLastError();
}

}  // namespace w4a16
