// Decode GEMV / tiny-N kernel on CUDA cores (memory-bound regime).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 2: the GEMV is memory
// bound; its design goals there are vectorised loads, unrolling to keep many
// loads in flight, the zero and scale of each int4 group kept close to the
// compute, and tiling both dimensions of the weight (rows and K) for
// parallelism.  On sm_100a that becomes:
//
//  * thread = one weight row; a warp covers 32 rows and reads 32 x 16 bytes
//    = 512 contiguous bytes of the packed layout per load instruction;
//  * each warp owns a range of whole groups along K and issues all loads of
//    up to two groups (8 x 16 B per thread) before any arithmetic;
//  * per-(row, group) scale and zero go straight to registers with the
//    weight loads (each is read once; there is no reuse for shared memory to
//    capture in this mapping);
//  * activations come through the read-only path, one broadcast 16-byte load
//    per 8 codes and token;
//  * split-K: warps of a CTA reduce through shared memory, and CTAs of a
//    thread-block cluster (up to 8 along K) reduce through distributed shared
//    memory into the cluster's rank-0 CTA, always in a fixed order, so the
//    result is deterministic (no atomics).
//  * products accumulate in fp32 with the mixed-precision fma.rn.f32.f16.
#include "w4a16_internal.cuh"

#include <algorithm>

namespace w4a16 {
namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kMaxCluster = 8;
constexpr int kBatchGroups = 2;  // groups whose loads are in flight together

__device__ __forceinline__ void fma_h2(float& acc, uint32_t w, uint32_t x) {
  asm("{\n\t.reg .f16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
      : "+f"(acc) : "r"(w), "r"(x));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads, NT == 1 ? 4 : 2)
gemv_kernel(const uint4* __restrict__ wq, const uint16_t* __restrict__ s_p,
            const uint8_t* __restrict__ z_p, const uint16_t* __restrict__ X,
            uint16_t* __restrict__ Y, int M, int K, int cl) {
  __shared__ float red[kGemvWarps][NT][32];
  __shared__ float cred[kMaxCluster][NT][32];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tile = blockIdx.x / cl;
  const int crank = blockIdx.x % cl;
  const int r0 = tile * 32;
  const int b = r0 / kRowBlock;
  const int r = (r0 % kRowBlock) + lane;   // row inside the 128-row block
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;

  if (cl > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // Whole groups along K: first split across the cluster, then across warps.
  const int ga = (kg * crank) / cl, gb = (kg * (crank + 1)) / cl;
  const int g0 = ga + ((gb - ga) * warp) / kGemvWarps;
  const int g1 = ga + ((gb - ga) * (warp + 1)) / kGemvWarps;

  float acc[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n] = 0.f;

  const uint4* wrow = wq + (size_t)b * kc_n * kRowBlock + r;   // chunk c at wrow[c * 128]
  const uint16_t* srow = s_p + (size_t)b * kg * kRowBlock + r;  // group g at srow[g * 128]
  const uint8_t* zrow = z_p + (size_t)b * kg * (kRowBlock / 2) + (r >> 1);
  const int zshift = (r & 1) * 4;

  for (int g = g0; g < g1; g += kBatchGroups) {
    const int ng = min(kBatchGroups, g1 - g);
    uint4 v[kBatchGroups * 4];
    uint16_t sv[kBatchGroups];
    uint32_t zv[kBatchGroups];
#pragma unroll
    for (int i = 0; i < kBatchGroups; ++i) {
      if (i < ng) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[i * 4 + j] = ldg_stream_v4(wrow + (size_t)((g + i) * 4 + j) * kRowBlock);
        sv[i] = __ldg(srow + (size_t)(g + i) * kRowBlock);
        zv[i] = __ldg(zrow + (size_t)(g + i) * (kRowBlock / 2));
      }
    }
#pragma unroll
    for (int i = 0; i < kBatchGroups; ++i) {
      if (i < ng) {
        GroupConsts gc = make_group_consts((zv[i] >> zshift) & 0xFu, sv[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kbase = ((g + i) * 4 + j) * kChunkK;
          uint32_t words[4] = {v[i * 4 + j].x, v[i * 4 + j].y, v[i * 4 + j].z, v[i * 4 + j].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            uint32_t h[4];
            dequant_word(words[t], gc, h);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              uint4 xv = ldg_ro_v4(X + (size_t)n * K + kbase + 8 * t);
              fma_h2(acc[n], h[0], xv.x);
              fma_h2(acc[n], h[1], xv.y);
              fma_h2(acc[n], h[2], xv.z);
              fma_h2(acc[n], h[3], xv.w);
            }
          }
        }
      }
    }
  }

#pragma unroll
  for (int n = 0; n < NT; ++n) red[warp][n][lane] = acc[n];
  __syncthreads();

  float tot[NT];
  if (warp == 0) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kGemvWarps; ++w) s += red[w][n][lane];
      tot[n] = s;
    }
  }

  if (cl > 1) {
    // Every CTA of the cluster has started once this wait returns, so its
    // shared memory may be written remotely.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (warp == 0) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint32_t local = smem_u32(&cred[crank][n][lane]);
        uint32_t remote;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(0));
        asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(remote), "f"(tot[n]) : "memory");
      }
    }
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (crank != 0 || warp != 0) return;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float s = 0.f;
      for (int c = 0; c < cl; ++c) s += cred[c][n][lane];
      tot[n] = s;
    }
  } else if (warp != 0) {
    return;
  }

  const int m = r0 + lane;
  if (m < M) {
#pragma unroll
    for (int n = 0; n < NT; ++n) Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(tot[n]));
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int NT>
cudaError_t launch_nt(const uint4* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int cl, int tiles, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * cl), 1, 1);
  cfg.blockDim = dim3(kGemvThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT>, wq, s_p, z_p, X, Y, M, K, cl);
}

}  // namespace

// Cluster size along K: enough CTAs to cover the SMs a few times over, while
// every warp keeps at least one whole group.
int gemv_cluster_size(int M, int K, int sms) {
  const int tiles = ceil_div(M, 32);
  const int kg = K / kGroup;
  int cl = 1;
  while (cl < kMaxCluster && tiles * cl < 3 * sms && kg / (2 * cl) >= kGemvWarps) cl *= 2;
  return cl;
}

cudaError_t launch_gemv(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                        const uint16_t* X, uint16_t* Y, int M, int K, int N,
                        cudaStream_t stream) {
  const int tiles = ceil_div(M, 32);
  const int cl = gemv_cluster_size(M, K, sm_count());
  const uint4* w4 = reinterpret_cast<const uint4*>(wq);
  for (int n0 = 0; n0 < N; n0 += kGemvMaxTokens) {
    const int nt = std::min(kGemvMaxTokens, N - n0);
    const uint16_t* Xn = X + (size_t)n0 * K;
    uint16_t* Yn = Y + (size_t)n0 * M;
    cudaError_t e;
    switch (nt) {
      case 1: e = launch_nt<1>(w4, scales, zeros, Xn, Yn, M, K, cl, tiles, stream); break;
      case 2: e = launch_nt<2>(w4, scales, zeros, Xn, Yn, M, K, cl, tiles, stream); break;
      case 3: e = launch_nt<3>(w4, scales, zeros, Xn, Yn, M, K, cl, tiles, stream); break;
      default: e = launch_nt<4>(w4, scales, zeros, Xn, Yn, M, K, cl, tiles, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace w4a16
