// Offline repack of canonical uint4 weights into the interleaved chunk layout,
// and the debug dequantisation that writes fp16 W from the packed buffers.
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.1: int4 weights with a scale and
// a zero per group of 128; section 3.3 item 1 stresses vectorised loads, which
// the 16-byte, row-interleaved chunks below serve.
#include "w4a16_internal.cuh"

namespace w4a16 {
namespace {

// Nibble position of the code at offset o (0..7) inside its 32-bit word:
// even offsets fill nibbles 0..3, odd offsets nibbles 4..7, so the pair
// (2i, 2i+1) sits in bits 4i and 16 + 4i.
__device__ __forceinline__ int nibble_of_offset(int o) { return (o & 1) ? 4 + (o >> 1) : (o >> 1); }

// One thread per 16-byte output chunk (block b, chunk column c, row r).
// mi > 0: the gate/up row order (packed_source_row).
__global__ void pack_weights_kernel(const uint8_t* __restrict__ q, int M, int K, int mi,
                                    uint4* __restrict__ wq_p, long long n_chunks) {
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_chunks) return;
  const int kc_n = K / kChunkK;
  int r = (int)(i % kRowBlock);
  long long t = i / kRowBlock;
  int c = (int)(t % kc_n);
  int b = (int)(t / kc_n);
  int m = packed_source_row(b, r, M, mi);
  uint32_t words[4] = {0u, 0u, 0u, 0u};
  if (m >= 0) {
    const uint8_t* src = q + (size_t)m * K + (size_t)c * kChunkK;
#pragma unroll
    for (int j = 0; j < kChunkK; ++j) {
      uint32_t code = src[j] & 0xFu;
      words[j >> 3] |= code << (4 * nibble_of_offset(j & 7));
    }
  }
  wq_p[i] = make_uint4(words[0], words[1], words[2], words[3]);
}

// One thread per (block b, group g, row pair rp): two scales and one zero byte.
__global__ void pack_meta_kernel(const uint16_t* __restrict__ scales,
                                 const uint8_t* __restrict__ zeros, int M, int K, int mi,
                                 uint16_t* __restrict__ s_p, uint8_t* __restrict__ z_p,
                                 long long n_pairs) {
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const int kg = K / kGroup;
  int rp = (int)(i % (kRowBlock / 2));
  long long t = i / (kRowBlock / 2);
  int g = (int)(t % kg);
  int b = (int)(t / kg);
  uint32_t zb = 0;
  long long base = (long long)(b * kg + g) * kRowBlock;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    int r = 2 * rp + h;
    int m = packed_source_row(b, r, M, mi);
    uint16_t s = 0;
    uint32_t z = 0;
    if (m >= 0) {
      s = scales[(size_t)m * kg + g];
      z = zeros[(size_t)m * kg + g] & 0xFu;
    }
    s_p[base + r] = s;
    zb |= z << (4 * h);
  }
  z_p[(long long)(b * kg + g) * (kRowBlock / 2) + rp] = (uint8_t)zb;
}

// One thread per packed chunk: the same dequant_word() the GEMM kernels use,
// written out as fp16 W[m][k].
__global__ void dequant_kernel(const uint4* __restrict__ wq_p, const uint16_t* __restrict__ s_p,
                               const uint8_t* __restrict__ z_p, int M, int K,
                               uint16_t* __restrict__ W, long long n_chunks) {
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_chunks) return;
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;
  int r = (int)(i % kRowBlock);
  long long t = i / kRowBlock;
  int c = (int)(t % kc_n);
  int b = (int)(t / kc_n);
  int m = b * kRowBlock + r;
  if (m >= M) return;
  int g = (c * kChunkK) / kGroup;
  const uint8_t* zblock = z_p + (size_t)(b * kg + g) * (kRowBlock / 2);
  GroupConsts gc = make_group_consts(zero_code(zblock, r), s_p[(size_t)(b * kg + g) * kRowBlock + r]);
  uint4 v = wq_p[i];
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint4* dst = reinterpret_cast<uint4*>(W + (size_t)m * K + (size_t)c * kChunkK);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4];
    dequant_word(w[j], gc, h);
    dst[j] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

}  // namespace

cudaError_t launch_pack(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                        int M, int K, uint8_t* wq_p, uint16_t* s_p, uint8_t* z_p,
                        cudaStream_t stream, int mi) {
  const int mb = ceil_div(M, kRowBlock);
  long long n_chunks = (long long)mb * (K / kChunkK) * kRowBlock;
  long long n_pairs = (long long)mb * (K / kGroup) * (kRowBlock / 2);
  const int threads = 256;
  pack_weights_kernel<<<(unsigned)((n_chunks + threads - 1) / threads), threads, 0, stream>>>(
      q, M, K, mi, reinterpret_cast<uint4*>(wq_p), n_chunks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pack_meta_kernel<<<(unsigned)((n_pairs + threads - 1) / threads), threads, 0, stream>>>(
      scales, zeros, M, K, mi, s_p, z_p, n_pairs);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           uint16_t* W, int M, int K, cudaStream_t stream) {
  const int mb = ceil_div(M, kRowBlock);
  long long n_chunks = (long long)mb * (K / kChunkK) * kRowBlock;
  const int threads = 256;
  dequant_kernel<<<(unsigned)((n_chunks + threads - 1) / threads), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(wq), scales, zeros, M, K, W, n_chunks);
  return cudaGetLastError();
}

}  // namespace w4a16
