// Decode GEMV / tiny-N kernel on CUDA cores (memory-bound regime).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 2: the GEMV is memory
// bound; its design goals there are vectorised loads, unrolling to keep many
// loads in flight, the zero and scale of each int4 group kept in shared
// memory, the vector read through a texture-like path, and tiling both
// dimensions of the weight (rows and K) for parallelism.  On sm_100a:
//
//  * a CTA owns one 128-row block of the packed weight and a range of whole
//    groups along K; a producer warp streams each group (8 KB of codes, 256 B
//    of scales, 64 B of zeros, contiguous in the packed layout) into a
//    6-stage shared-memory ring with bulk asynchronous copies, so tens of KB
//    per CTA are in flight without holding registers;
//  * the CTA's slice of the activations is staged once in shared memory and
//    read back as broadcast 16-byte loads;
//  * two consumer warpgroups take alternate groups; thread = one weight row;
//    the exact in-register dequant (dequant_word) feeds fma.rn.f32.f16 into
//    four independent fp32 chains per token;
//  * split-K: the two warpgroups reduce through shared memory, and CTAs of a
//    thread-block cluster (up to 8 along K) through distributed shared memory
//    into the cluster's rank-0 CTA, in a fixed order (deterministic, no
//    atomics);
//  * every mbarrier wait is bounded (device status word on expiry).
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

#include <algorithm>

namespace w4a16 {

__device__ int g_gemv_status = 0;

namespace {

constexpr int kGvHalves = 2;                          // consumer warpgroups (alternate groups)
constexpr int kGvConsumerWarps = 4 * kGvHalves;
constexpr int kGvProducerWarp = kGvConsumerWarps;
constexpr int kGvThreads = (kGvConsumerWarps + 1) * 32;
constexpr int kGvWBytes = 4 * kRowBlock * 16;         // one group of 128 rows: 8 KB
constexpr int kGvStageBytes = kGvWBytes + kRowBlock * 2 + kRowBlock / 2;   // + scales + zeros
constexpr int kGvStages = 6;                          // multiple of kGvHalves
constexpr int kMaxCluster = 8;
constexpr int kMaxXSmem = 64 * 1024;                  // largest staged activation slice
static_assert(kGvStages % kGvHalves == 0, "stage ring");

__device__ __forceinline__ void fma_h2(float& acc, uint32_t w, uint32_t x) {
  asm("{\n\t.reg .f16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
      : "+f"(acc) : "r"(w), "r"(x));
}

struct GvLayout {
  int x_off, red_off, cred_off, bar_off, total;
};

__host__ __device__ inline GvLayout gv_layout(int nt, int gspan, int cl) {
  GvLayout L;
  L.x_off = kGvStages * kGvStageBytes;
  L.red_off = L.x_off + nt * gspan * kGroup * 2;
  L.cred_off = L.red_off + kGvHalves * nt * kRowBlock * 4;
  L.bar_off = L.cred_off + (cl > 1 ? cl * nt * kRowBlock * 4 : 0);
  L.total = L.bar_off + 8 * (2 * kGvStages + 1) + 16;
  return L;
}

template <int NT, int kEpi>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(const uint8_t* __restrict__ wq, const uint16_t* __restrict__ s_p,
            const uint8_t* __restrict__ z_p, const uint16_t* __restrict__ X,
            uint16_t* __restrict__ Y, int M, int K, int cl, OutMap om) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int kg = K / kGroup;
  const int kc_n = K / kChunkK;
  const int gspan = ceil_div(kg, cl);
  const GvLayout L = gv_layout(NT, gspan, cl);
  uint4* xs = reinterpret_cast<uint4*>(smem + L.x_off);
  float* red = reinterpret_cast<float*>(smem + L.red_off);     // [halves][NT][128]
  float* cred = reinterpret_cast<float*>(smem + L.cred_off);   // [cl][NT][128], rank 0 only
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + kGvStages;
  uint64_t* xbar = empty + kGvStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x / cl;
  const int crank = blockIdx.x % cl;
  const int ga = (kg * crank) / cl, gb = (kg * (crank + 1)) / cl;
  const int ng = gb - ga;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGvStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 4);              // the 4 warps of one consumer half
    }
    ptx::mbar_init(xbar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (cl > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  float tot[NT];
  if (warp == kGvProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ng > 0) {
      ptx::mbar_arrive_expect_tx(xbar, (uint32_t)(NT * ng * kGroup * 2));
      for (int n = 0; n < NT; ++n)
        ptx::bulk_load(reinterpret_cast<uint8_t*>(xs) + n * ng * kGroup * 2,
                       X + (size_t)n * K + (size_t)ga * kGroup, (uint32_t)(ng * kGroup * 2), xbar);
      const uint8_t* wblk = wq + (size_t)b * kc_n * kRowBlock * 16;
      const uint16_t* sblk = s_p + (size_t)b * kg * kRowBlock;
      const uint8_t* zblk = z_p + (size_t)b * kg * (kRowBlock / 2);
      int last = -1;
      for (int i = 0; i < ng; ++i) {
        const int st = i % kGvStages;
        const uint32_t ph = (uint32_t)((i / kGvStages) & 1);
        if (!wait_bar(&empty[st], ph ^ 1, abort_flag, &g_gemv_status)) break;
        uint8_t* dst = smem + st * kGvStageBytes;
        const int g = ga + i;
        ptx::mbar_arrive_expect_tx(&full[st], kGvStageBytes);
        ptx::bulk_load(dst, wblk + (size_t)g * kGvWBytes, kGvWBytes, &full[st]);
        ptx::bulk_load(dst + kGvWBytes, sblk + (size_t)g * kRowBlock, kRowBlock * 2, &full[st]);
        ptx::bulk_load(dst + kGvWBytes + kRowBlock * 2, zblk + (size_t)g * (kRowBlock / 2), kRowBlock / 2,
                       &full[st]);
        last = i;
      }
      // Drain: every copy issued into this CTA's shared memory has landed.
      for (int i = (last - kGvStages + 1 > 0 ? last - kGvStages + 1 : 0); i <= last; ++i)
        wait_bar(&full[i % kGvStages], (uint32_t)((i / kGvStages) & 1), abort_flag, &g_gemv_status, false);
      wait_bar(xbar, 0, abort_flag, &g_gemv_status, false);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- consumers
    // Thread = weight row r of block b; consumer half h takes groups
    // i = h, h + 2, ...; four independent fp32 chains per token.
    const int h = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int t = 0; t < 4; ++t) acc[n][t] = 0.f;
    bool ok = ng == 0 || wait_bar_warp(xbar, 0, abort_flag, &g_gemv_status);
    for (int i = h; ok && i < ng; i += kGvHalves) {
      const int st = i % kGvStages;
      const uint32_t ph = (uint32_t)((i / kGvStages) & 1);
      if (!wait_bar_warp(&full[st], ph, abort_flag, &g_gemv_status)) break;
      const uint8_t* src = smem + st * kGvStageBytes;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(src + j * kRowBlock * 16 + r * 16);
      const uint16_t sv = reinterpret_cast<const uint16_t*>(src + kGvWBytes)[r];
      const uint32_t zb = src[kGvWBytes + kRowBlock * 2 + (r >> 1)];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[st]);
      const GroupConsts gc = make_group_consts((zb >> ((r & 1) * 4)) & 0xFu, sv);
      // The group's activations: token n at xg + n * ng * 16, then fixed offsets.
      const uint4* xg = xs + i * (kGroup / 8);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t words[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          uint32_t hw[4];
          dequant_word(words[t], gc, hw);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint4 xv = xg[n * ng * (kGroup / 8) + j * 4 + t];
            fma_h2(acc[n][t], hw[0], xv.x);
            fma_h2(acc[n][t], hw[1], xv.y);
            fma_h2(acc[n][t], hw[2], xv.z);
            fma_h2(acc[n][t], hw[3], xv.w);
          }
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n)
      red[(h * NT + n) * kRowBlock + r] = (acc[n][0] + acc[n][1]) + (acc[n][2] + acc[n][3]);
  }
  __syncthreads();

  const int r = threadIdx.x;   // rows for the reduction: threads 0..127
  // The fused form's destination and bias of row m, loaded before the
  // reductions so the load overlaps them.
  RowDst dst = {};
  if constexpr (kEpi == kEpiQkv) {
    const int m = b * kRowBlock + r;
    if (r < kRowBlock && crank == 0 && m < M) dst = row_dst(om, M, m);
  }
  if (r < kRowBlock) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sum = 0.f;
#pragma unroll
      for (int h = 0; h < kGvHalves; ++h) sum += red[(h * NT + n) * kRowBlock + r];
      tot[n] = sum;
    }
  }

  if (cl > 1) {
    // Every CTA of the cluster has started once this wait returns, so its
    // shared memory may be written remotely.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (r < kRowBlock) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint32_t local = ptx::smem_addr(&cred[(crank * NT + n) * kRowBlock + r]);
        uint32_t remote;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(0));
        asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(remote), "f"(tot[n]) : "memory");
      }
    }
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (crank != 0 || r >= kRowBlock) return;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sum = 0.f;
      for (int c = 0; c < cl; ++c) sum += cred[(c * NT + n) * kRowBlock + r];
      tot[n] = sum;
    }
  } else if (r >= kRowBlock) {
    return;
  }

  const int m = b * kRowBlock + r;
  if constexpr (kEpi == kEpiGateUp) {
    // Threads 0..127 are whole warps here: the gate/up pairing shuffles.
#pragma unroll
    for (int n = 0; n < NT; ++n) store_gate_up(om, b, r, n, tot[n], true);
  } else if (m < M) {
    if constexpr (kEpi == kEpiQkv) {
#pragma unroll
      for (int n = 0; n < NT; ++n) store_row(dst, om.bias != nullptr, n, tot[n]);
    } else {
#pragma unroll
      for (int n = 0; n < NT; ++n) Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(tot[n]));
    }
  }
}

template <int NT, int kEpi>
cudaError_t launch_nt(const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int cl, cudaStream_t stream, const OutMap& om) {
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemv_kernel<NT, kEpi>), 200 * 1024, smem_set);
  if (e != cudaSuccess) return e;
  const int blocks = ceil_div(M, kRowBlock);
  const GvLayout L = gv_layout(NT, ceil_div(K / kGroup, cl), cl);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(blocks * cl), 1, 1);
  cfg.blockDim = dim3(kGvThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, kEpi>, wq, s_p, z_p, X, Y, M, K, cl, om);
}

}  // namespace

// Cluster size along K (1..8), from the measured LLaMA-7B N = 1 shapes:
// all CTAs resident in one wave (kGvCtasPerSm per SM, set by the shared
// memory of one CTA), and at least 2.5 CTAs per SM on average when the shape
// allows it (fewer warps per SM hide the shared-memory and FMA latencies
// badly); among those the smallest busiest-SM share of groups,
// ceil(CTAs / SMs) x ceil(groups / cluster), then the smaller cluster.  When
// no cluster reaches 2.5 CTAs per SM, the most CTAs.  The staged activation
// slice must fit.
int gemv_cluster_size(int M, int K, int sms, int nt) {
  constexpr int kGvCtasPerSm = 4;
  const int blocks = ceil_div(M, kRowBlock);
  const int kg = K / kGroup;
  int best = 0;
  long long best_key[3] = {0, 0, 0};
  for (int cl = 1; cl <= kMaxCluster && cl <= kg; ++cl) {
    if (nt * ceil_div(kg, cl) * kGroup * 2 > kMaxXSmem) continue;
    const long long ctas = (long long)blocks * cl;
    if (cl > 1 && ctas > (long long)kGvCtasPerSm * sms) continue;
    const bool dense = 2 * ctas >= 5LL * sms;
    const long long load = (long long)ceil_div((int)ctas, sms) * ceil_div(kg, cl);
    const long long key[3] = {dense ? 0 : 1, dense ? load : -ctas, cl};
    if (best == 0 || key[0] < best_key[0] || (key[0] == best_key[0] && (key[1] < best_key[1] ||
        (key[1] == best_key[1] && key[2] < best_key[2])))) {
      best = cl;
      for (int i = 0; i < 3; ++i) best_key[i] = key[i];
    }
  }
  return best > 0 ? best : kMaxCluster;
}

cudaError_t launch_gemv(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                        const uint16_t* X, uint16_t* Y, int M, int K, int N,
                        cudaStream_t stream, const OutMap* om) {
  for (int n0 = 0; n0 < N; n0 += kGemvMaxTokens) {
    const int nt = std::min(kGemvMaxTokens, N - n0);
    const int cl = gemv_cluster_size(M, K, num_sms(), nt);
    if (nt * ceil_div(K / kGroup, cl) * kGroup * 2 > kMaxXSmem) return cudaErrorNotSupported;
    const uint16_t* Xn = X + (size_t)n0 * K;
    uint16_t* Yn = om ? nullptr : Y + (size_t)n0 * M;
    // The fused outputs of tokens n0 .. n0 + nt - 1: each segment moves by
    // n0 of its own rows.
    OutMap on = {};
    if (om) {
      on = *om;
      if (om->kind == kEpiGateUp) {
        on.h = om->h + (size_t)n0 * om->mi;
      } else {
        on.y0 = om->y0 + (size_t)n0 * om->end0;
        on.y1 = om->y1 + (size_t)n0 * (om->end1 - om->end0);
        on.y2 = om->y2 + (size_t)n0 * (M - om->end1);
      }
    }
    const int kind = om ? om->kind : kEpiPlain;
    cudaError_t e;
#define W4A16_GEMV_NT(EPI)                                                                          \
    switch (nt) {                                                                                     \
      case 1: e = launch_nt<1, EPI>(wq, scales, zeros, Xn, Yn, M, K, cl, stream, on); break;          \
      case 2: e = launch_nt<2, EPI>(wq, scales, zeros, Xn, Yn, M, K, cl, stream, on); break;          \
      case 3: e = launch_nt<3, EPI>(wq, scales, zeros, Xn, Yn, M, K, cl, stream, on); break;          \
      default: e = launch_nt<4, EPI>(wq, scales, zeros, Xn, Yn, M, K, cl, stream, on); break;         \
    }
    if (kind == kEpiGateUp) {
      W4A16_GEMV_NT(kEpiGateUp)
    } else if (kind == kEpiQkv) {
      W4A16_GEMV_NT(kEpiQkv)
    } else {
      W4A16_GEMV_NT(kEpiPlain)
    }
#undef W4A16_GEMV_NT
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t read_and_clear_gemv_status(int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_gemv_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_gemv_status, &zero, sizeof(int));
}

}  // namespace w4a16
