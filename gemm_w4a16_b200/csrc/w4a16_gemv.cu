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
//  * each warp owns a range of whole groups along K and walks it with the
//    next group's loads (4 x 16 B + scale + zero per thread) in flight while
//    the current group is dequantised: double-buffered registers;
//  * per-(row, group) scale and zero go straight to registers with the
//    weight loads (each is read once; there is no reuse for shared memory to
//    capture in this mapping);
//  * the CTA's slice of the activations is staged once in shared memory
//    (the analogue of the page's image-typed vector reads) and read back as
//    broadcast 16-byte loads, one per 8 codes and token;
//  * split-K: warps of a CTA reduce through shared memory, and CTAs of a
//    thread-block cluster (up to 8 along K) reduce through distributed shared
//    memory into the cluster's rank-0 CTA, always in a fixed order, so the
//    result is deterministic (no atomics).
//  * products accumulate in fp32 with the mixed-precision fma.rn.f32.f16.
#include "w4a16_internal.cuh"

#include <algorithm>

namespace w4a16 {
namespace {

constexpr int kGemvWarps = 4;                 // warps splitting K inside a CTA
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kRowsPerCta = 32;               // one row per lane
constexpr int kMaxCluster = 8;
constexpr int kMaxXSmem = 96 * 1024;          // largest staged activation slice

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

// One group (128 codes) of one row: four 16-byte chunks plus its scale and
// zero byte.
struct GroupRegs {
  uint4 v[4];
  uint16_t s;
  uint32_t z;
};

template <int NT>
__global__ void __launch_bounds__(kGemvThreads, NT == 1 ? 8 : 4)
gemv_kernel(const uint4* __restrict__ wq, const uint16_t* __restrict__ s_p,
            const uint8_t* __restrict__ z_p, const uint16_t* __restrict__ X,
            uint16_t* __restrict__ Y, int M, int K, int cl) {
  extern __shared__ uint4 xs[];                 // [NT][kspan] fp16, 8 per uint4
  __shared__ float red[kGemvWarps][NT][32];
  __shared__ float cred[kMaxCluster][NT][32];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tile = blockIdx.x / cl;
  const int crank = blockIdx.x % cl;
  const int r0 = tile * kRowsPerCta;
  const int b = r0 / kRowBlock;
  const int r = (r0 % kRowBlock) + lane;   // row inside the 128-row block
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;

  if (cl > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // Whole groups along K: first split across the cluster, then across warps.
  const int ga = (kg * crank) / cl, gb = (kg * (crank + 1)) / cl;
  const int g0 = ga + ((gb - ga) * warp) / kGemvWarps;
  const int g1 = ga + ((gb - ga) * (warp + 1)) / kGemvWarps;
  const int kspan8 = (gb - ga) * (kGroup / 8);   // uint4 per token in the slice

  const uint4* wrow = wq + (size_t)b * kc_n * kRowBlock + r;   // chunk c at wrow[c * 128]
  const uint16_t* srow = s_p + (size_t)b * kg * kRowBlock + r;  // group g at srow[g * 128]
  const uint8_t* zrow = z_p + (size_t)b * kg * (kRowBlock / 2) + (r >> 1);
  const int zshift = (r & 1) * 4;

  auto load_group = [&](int g, GroupRegs& gr) {
#pragma unroll
    for (int j = 0; j < 4; ++j) gr.v[j] = ldg_stream_v4(wrow + (size_t)(g * 4 + j) * kRowBlock);
    gr.s = __ldg(srow + (size_t)g * kRowBlock);
    gr.z = __ldg(zrow + (size_t)g * (kRowBlock / 2));
  };

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[n][t] = 0.f;

  auto compute_group = [&](int g, const GroupRegs& gr) {
    const GroupConsts gc = make_group_consts((gr.z >> zshift) & 0xFu, gr.s);
    const int xo = (g - ga) * (kGroup / 8);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t words[4] = {gr.v[j].x, gr.v[j].y, gr.v[j].z, gr.v[j].w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t h[4];
        dequant_word(words[t], gc, h);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 xv = xs[n * kspan8 + xo + j * 4 + t];
          fma_h2(acc[n][t], h[0], xv.x);
          fma_h2(acc[n][t], h[1], xv.y);
          fma_h2(acc[n][t], h[2], xv.z);
          fma_h2(acc[n][t], h[3], xv.w);
        }
      }
    }
  };

  // First group's loads go out before the activation slice is staged, so
  // their latency overlaps the staging.
  GroupRegs ga_regs, gb_regs;
  if (g0 < g1) load_group(g0, ga_regs);
  {
    const uint4* xsrc = reinterpret_cast<const uint4*>(X);
    const int k8 = K / 8;
    for (int i = threadIdx.x; i < NT * kspan8; i += kGemvThreads) {
      const int n = i / kspan8, o = i - n * kspan8;
      xs[i] = __ldg(xsrc + (size_t)n * k8 + ga * (kGroup / 8) + o);
    }
  }
  __syncthreads();

  // Double-buffered walk over the warp's groups: the next group's loads are
  // in flight while the current one is dequantised and multiplied.
  for (int g = g0; g < g1; g += 2) {
    if (g + 1 < g1) load_group(g + 1, gb_regs);
    compute_group(g, ga_regs);
    if (g + 1 < g1) {
      if (g + 2 < g1) load_group(g + 2, ga_regs);
      compute_group(g + 1, gb_regs);
    }
  }

#pragma unroll
  for (int n = 0; n < NT; ++n) red[warp][n][lane] = (acc[n][0] + acc[n][1]) + (acc[n][2] + acc[n][3]);
  __syncthreads();

  float tot[NT];
  if (warp == 0) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kGemvWarps; ++w) sum += red[w][n][lane];
      tot[n] = sum;
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
      float sum = 0.f;
      for (int c = 0; c < cl; ++c) sum += cred[c][n][lane];
      tot[n] = sum;
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

int x_smem_bytes(int K, int cl, int nt) {
  const int kg = K / kGroup;
  return nt * ceil_div(kg, cl) * kGroup * 2;
}

template <int NT>
cudaError_t launch_nt(const uint4* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int cl, int tiles, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxXSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * cl), 1, 1);
  cfg.blockDim = dim3(kGemvThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)x_smem_bytes(K, cl, NT);
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

// Cluster size along K.  One wave of CTAs (every CTA resident at once) with as
// many CTAs as fit, while each warp keeps at least two whole groups so the
// double-buffered loads have something to overlap; larger if the activation
// slice would not fit in shared memory.
int gemv_cluster_size(int M, int K, int sms, int nt) {
  const int tiles = ceil_div(M, kRowsPerCta);
  const int kg = K / kGroup;
  const int resident = sms * (nt == 1 ? 8 : 4);
  int cl = 1;
  while (cl < kMaxCluster && tiles * cl * 2 <= resident && kg / (2 * cl) >= 2 * kGemvWarps) cl *= 2;
  while (cl < kMaxCluster && x_smem_bytes(K, cl, nt) > kMaxXSmem) cl *= 2;
  return cl;
}

cudaError_t launch_gemv(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                        const uint16_t* X, uint16_t* Y, int M, int K, int N,
                        cudaStream_t stream) {
  const int tiles = ceil_div(M, kRowsPerCta);
  const uint4* w4 = reinterpret_cast<const uint4*>(wq);
  for (int n0 = 0; n0 < N; n0 += kGemvMaxTokens) {
    const int nt = std::min(kGemvMaxTokens, N - n0);
    const int cl = gemv_cluster_size(M, K, sm_count(), nt);
    if (x_smem_bytes(K, cl, nt) > kMaxXSmem) return cudaErrorNotSupported;
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
