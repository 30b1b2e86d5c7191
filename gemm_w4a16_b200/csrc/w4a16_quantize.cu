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
// One warp per (row, group): lane l reads the group's weights 4l .. 4l + 3
// (8 bytes; the warp reads the group's 256 contiguous bytes), the warp finds
// the minimum and maximum by shuffles, and each lane writes its four codes as
// one 32-bit store.  Bound by HBM: 2 bytes read and 1 byte written per weight.
#include "w4a16_internal.cuh"

namespace w4a16 {

namespace {

constexpr int kQWarpsPerBlock = 8;

__device__ __forceinline__ float fp16_bits_to_float(uint32_t bits) {
  return __half2float(__ushort_as_half((unsigned short)(bits & 0xFFFFu)));
}

__global__ void __launch_bounds__(kQWarpsPerBlock * 32)
quantize_kernel(const uint16_t* __restrict__ W, int M, int K, uint8_t* __restrict__ q,
                uint16_t* __restrict__ s_out, uint8_t* __restrict__ z_out) {
  const int kg = K / kGroup;
  const long long unit = (long long)blockIdx.x * kQWarpsPerBlock + (threadIdx.x >> 5);
  if (unit >= (long long)M * kg) return;             // whole warps leave together
  const int lane = threadIdx.x & 31;
  const int m = (int)(unit / kg);
  const int g = (int)(unit - (long long)m * kg);
  const size_t base = (size_t)m * K + (size_t)g * kGroup + 4 * lane;

  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(W + base));
  float v[4];
  v[0] = fp16_bits_to_float(raw.x);
  v[1] = fp16_bits_to_float(raw.x >> 16);
  v[2] = fp16_bits_to_float(raw.y);
  v[3] = fp16_bits_to_float(raw.y >> 16);

  float lo = 0.0f, hi = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo = fminf(lo, v[i]);
    hi = fmaxf(hi, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }

  float r = __fsub_rn(hi, lo);
  const float r_min = 6.103515625e-05f;             // 2^-14
  if (!(r >= r_min)) r = r_min;
  const __half s16 = __float2half_rn(__fdiv_rn(r, 15.0f));
  const float f = __fdiv_rn(1.0f, __half2float(s16));
  const float zf = fminf(fmaxf(rintf(__fmul_rn(-lo, f)), 0.0f), 15.0f);

  uint32_t codes = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float qf = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(v[i], f)), zf), 0.0f), 15.0f);
    codes |= (uint32_t)qf << (8 * i);
  }
  *reinterpret_cast<uint32_t*>(q + base) = codes;
  if (lane == 0) {
    s_out[(size_t)m * kg + g] = __half_as_ushort(s16);
    z_out[(size_t)m * kg + g] = (uint8_t)zf;
  }
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int M, int K, uint8_t* q, uint16_t* scales, uint8_t* zeros,
                            cudaStream_t stream) {
  const long long units = (long long)M * (K / kGroup);
  const long long blocks = (units + kQWarpsPerBlock - 1) / kQWarpsPerBlock;
  if (blocks > 0x7fffffffLL) return cudaErrorNotSupported;
  quantize_kernel<<<(unsigned)blocks, kQWarpsPerBlock * 32, 0, stream>>>(W, M, K, q, scales, zeros);
  return cudaGetLastError();
}

}  // namespace w4a16
