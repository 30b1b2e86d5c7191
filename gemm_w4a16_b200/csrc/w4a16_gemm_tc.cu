// Large-N W4A16 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1: with many tokens the
// GEMM is compute bound; it gets its own tiling, with the operands staged in
// shared memory to cut global traffic.  On sm_100a the tile is 128 weight
// rows x BN tokens, K in stages of 64:
//
//   warp 4        producer: per stage one TMA tile of X (BN x 64 fp16, 128-byte
//                 swizzle, rows past N zero-filled) and bulk copies of the
//                 stage's packed codes (128 rows x 64 codes = 4 KB, contiguous
//                 in the packed layout) and of its group's scales and zeros.
//   warps 8..23   dequantisers: four groups of four warps take the stages in
//                 turn (four stages in flight); one weight row per thread
//                 (warp w serves TMEM lanes 32 (w % 4) ..), 64 codes; the exact
//                 in-register dequant (the same one the GEMV uses) writes
//                 fp16 W straight into tensor memory with tcgen05.st, where
//                 it is the MMA's A operand -- W never round-trips through
//                 shared memory, so shared-memory bandwidth is left to X.
//   warp 5        MMA issuer: tcgen05.mma kind::f16 (A from TMEM, B = X from
//                 shared memory, fp32 accumulator in TMEM), 4 MMAs of K = 16
//                 per stage; tcgen05.commit releases the stage, the A slot
//                 and, at the end of a tile, the accumulator.
//   warps 0..3    epilogue: tcgen05.ld of the fp32 accumulator, one RNE
//                 conversion to fp16, stores of Y[n][m].
//
// Persistent CTAs (one per SM) walk the tile list round-robin; accumulators
// are double-buffered in TMEM when they fit so the epilogue of one tile
// overlaps the main loop of the next.  Every mbarrier wait is bounded: on
// expiry the kernel records a timeout in a device status word, stops issuing,
// drains its copies and MMAs, frees TMEM and returns.
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace w4a16 {

__device__ int g_tc_status = 0;

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
// Warp roles: 0..3 epilogue (TMEM lane quadrants 0..3), 4 producer, 5 MMA
// issuer and TMEM owner, 6..7 idle, 8.. dequantiser groups of 4 warps.
constexpr int kDqGroups = 4;                     // stages dequantised concurrently
constexpr int kFirstDqWarp = 8;
constexpr int kThreads = (kFirstDqWarp + 4 * kDqGroups) * 32;
constexpr int kWBytes = kBM * kBK / 2;       // packed codes of one stage
constexpr int kSBytes = kBM * 2;             // scales of the stage's group
constexpr int kZBytes = kBM / 2;             // zeros of the stage's group
constexpr int kAColsPerSlot = kBK / 2;       // 64 fp16 = 32 columns

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

template <int BN>
struct Cfg {
  static constexpr int kXBytes = BN * kBK * 2;
  static constexpr int kStageBytes = round_up(kXBytes + kWBytes + kSBytes + kZBytes, 1024);
  // As many stages as fit in about 200 KB (a multiple of the dequantiser
  // group count, at most 24): the ring is what keeps copies in flight.
  static constexpr int kStagesFit = (200 * 1024 / kStageBytes) / kDqGroups * kDqGroups;
  static constexpr int kStages = kStagesFit < 24 ? kStagesFit : 24;
  static constexpr int kAccBufs = (2 * BN + kDqGroups * kAColsPerSlot <= 512) ? 2 : 1;
  static constexpr int kACol0 = kAccBufs * BN;
  // TMEM A slots (32 columns each): all the columns the accumulators leave,
  // a multiple of the dequantiser group count, at most 12.  The slot ring is
  // what lets dequantisation run ahead of MMA completion.
  static constexpr int kASlotsFit = (512 - kACol0) / kAColsPerSlot / kDqGroups * kDqGroups;
  static constexpr int kASlots = kASlotsFit < 12 ? kASlotsFit : 12;
  static constexpr int kColsUsed = kACol0 + kASlots * kAColsPerSlot;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static constexpr uint32_t kTx = kXBytes + kWBytes + kSBytes + kZBytes;
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kBM, BN);
  // Shared memory: stages, then barriers and the TMEM address.  At least
  // 120 KB is requested so that one CTA owns an SM (and all of its TMEM).
  static constexpr int kBarBytes = 8 * (2 * kStages + 2 * kASlots + 2 * kAccBufs + 1) + 16;
  static constexpr int kSmemUsed = kStages * kStageBytes + kBarBytes + 1024;
  static constexpr int kSmemBytes = kSmemUsed < 120 * 1024 ? 120 * 1024 : kSmemUsed;
  static_assert(kStages >= kDqGroups && kStages % kDqGroups == 0, "stage ring");
  static_assert(kASlots >= kDqGroups && kASlots % kDqGroups == 0, "TMEM A slot ring");
  static_assert(kColsUsed <= 512, "TMEM overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
};

struct Shared {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* a_full;
  uint64_t* a_empty;
  uint64_t* acc_full;
  uint64_t* acc_empty;
  uint64_t* drain;
  uint32_t* tmem_ptr;
  volatile int* abort_flag;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ wq,
               const uint16_t* __restrict__ s_p, const uint8_t* __restrict__ z_p,
               uint16_t* __restrict__ Y, int M, int K, int N) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  Shared sh;
  sh.full = bars;
  sh.empty = sh.full + C::kStages;
  sh.a_full = sh.empty + C::kStages;
  sh.a_empty = sh.a_full + C::kASlots;
  sh.acc_full = sh.a_empty + C::kASlots;
  sh.acc_empty = sh.acc_full + C::kAccBufs;
  sh.drain = sh.acc_empty + C::kAccBufs;
  sh.tmem_ptr = reinterpret_cast<uint32_t*>(sh.drain + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_ptr + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt_n = ceil_div(M, kBM);
  const int nt_n = ceil_div(N, BN);
  const int tiles = mt_n * nt_n;
  const int ks_n = K / kBK;
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      ptx::mbar_init(&sh.full[i], 1);
      ptx::mbar_init(&sh.empty[i], 4 + 1);     // 4 dequant warps + 1 MMA commit
    }
    for (int i = 0; i < C::kASlots; ++i) {
      ptx::mbar_init(&sh.a_full[i], 4);
      ptx::mbar_init(&sh.a_empty[i], 1);
    }
    for (int i = 0; i < C::kAccBufs; ++i) {
      ptx::mbar_init(&sh.acc_full[i], 1);
      ptx::mbar_init(&sh.acc_empty[i], 4);
    }
    ptx::mbar_init(sh.drain, 1);
    *sh.abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == 5) {
    ptx::tmem_alloc(sh.tmem_ptr, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sh.tmem_ptr;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int mt = t % mt_n, nt = t / mt_n;
        const uint8_t* wblk = wq + (size_t)mt * kc_n * kRowBlock * 16;
        for (int ks = 0; ks < ks_n; ++ks) {
          if (!wait_bar(&sh.empty[s], ph ^ 1, sh.abort_flag, &g_tc_status)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          ptx::mbar_arrive_expect_tx(&sh.full[s], C::kTx);
          ptx::tma_load_2d(st, &tmap_x, &sh.full[s], ks * kBK, nt * BN);
          ptx::bulk_load(st + C::kXBytes, wblk + (size_t)ks * 2 * kRowBlock * 16, kWBytes, &sh.full[s]);
          const int g = ks / 2;
          ptx::bulk_load(st + C::kXBytes + kWBytes, s_p + ((size_t)mt * kg + g) * kRowBlock, kSBytes,
                         &sh.full[s]);
          ptx::bulk_load(st + C::kXBytes + kWBytes + kSBytes,
                         z_p + ((size_t)mt * kg + g) * (kRowBlock / 2), kZBytes, &sh.full[s]);
          issued_mask |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == C::kStages) { s = 0; ph ^= 1; }
        }
      }
      // Drain: every copy issued into this CTA's shared memory has landed.
      for (int i = 0; i < C::kStages; ++i)
        if (issued_mask & (1u << i)) wait_bar(&sh.full[i], (issued_par >> i) & 1u, sh.abort_flag, &g_tc_status, false);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, a = 0, b = 0;
      uint32_t ph = 0, aph = 0, bph = 0;
      bool ok = true;
      const uint32_t x_base = ptx::smem_addr(smem);
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        if (!wait_bar(&sh.acc_empty[b], bph ^ 1, sh.abort_flag, &g_tc_status)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * BN;
        for (int ks = 0; ks < ks_n; ++ks) {
          if (!wait_bar(&sh.full[s], ph, sh.abort_flag, &g_tc_status) || !wait_bar(&sh.a_full[a], aph, sh.abort_flag, &g_tc_status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t xs = x_base + s * C::kStageBytes;
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j) {
            ptx::mma_ts_f16(d_tmem, tmem + C::kACol0 + a * kAColsPerSlot + 8 * j,
                            ptx::smem_desc_sw128(xs + 32 * j), C::kIdesc, (ks | j) != 0);
          }
          ptx::mma_commit(&sh.empty[s]);
          ptx::mma_commit(&sh.a_empty[a]);
          if (++s == C::kStages) { s = 0; ph ^= 1; }
          if (++a == C::kASlots) { a = 0; aph ^= 1; }
        }
        if (!ok) break;
        ptx::mma_commit(&sh.acc_full[b]);
        if (++b == C::kAccBufs) { b = 0; bph ^= 1; }
      }
      // Drain: all MMAs issued by this thread have completed.
      ptx::mma_commit(sh.drain);
      wait_bar(sh.drain, 0, sh.abort_flag, &g_tc_status, false);
    }
  } else if (warp >= kFirstDqWarp) {
    // -------------------------------------------------------- dequantisers
    // Group gi takes every kDqGroups-th stage of this CTA's sequence (so
    // kDqGroups stages are in flight at once); stage i goes to TMEM A slot
    // i % kASlots; each thread dequantises the 64 codes of one row.
    const int gi = (warp - kFirstDqWarp) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t a_lane = tmem + ((uint32_t)(quad * 32) << 16) + C::kACol0;
    const int my_tiles = (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const long long n_stages = (long long)my_tiles * ks_n;
    for (long long i = gi; i < n_stages; i += kDqGroups) {
      const int s = (int)(i % C::kStages);
      const uint32_t ph = (uint32_t)((i / C::kStages) & 1);
      const int a = (int)(i % C::kASlots);
      const uint32_t aph = (uint32_t)((i / C::kASlots) & 1);
      if (!wait_bar_warp(&sh.full[s], ph, sh.abort_flag, &g_tc_status)) break;
      const uint8_t* st = smem + s * C::kStageBytes;
      const uint4 v0 = *reinterpret_cast<const uint4*>(st + C::kXBytes + row * 16);
      const uint4 v1 = *reinterpret_cast<const uint4*>(st + C::kXBytes + kRowBlock * 16 + row * 16);
      const uint16_t sv = reinterpret_cast<const uint16_t*>(st + C::kXBytes + kWBytes)[row];
      const uint32_t zb = st[C::kXBytes + kWBytes + kSBytes + (row >> 1)];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.empty[s]);
      const GroupConsts gc = make_group_consts((zb >> ((row & 1) * 4)) & 0xFu, sv);
      uint32_t h[32];
      dequant_word(v0.x, gc, &h[0]);
      dequant_word(v0.y, gc, &h[4]);
      dequant_word(v0.z, gc, &h[8]);
      dequant_word(v0.w, gc, &h[12]);
      dequant_word(v1.x, gc, &h[16]);
      dequant_word(v1.y, gc, &h[20]);
      dequant_word(v1.z, gc, &h[24]);
      dequant_word(v1.w, gc, &h[28]);
      if (!wait_bar_warp(&sh.a_empty[a], aph ^ 1, sh.abort_flag, &g_tc_status)) break;
      ptx::tc_fence_after();
      ptx::tmem_st_x32(a_lane + a * kAColsPerSlot, h);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.a_full[a]);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    int b = 0;
    uint32_t bph = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int mt = t % mt_n, nt = t / mt_n;
      if (!wait_bar_warp(&sh.acc_full[b], bph, sh.abort_flag, &g_tc_status)) break;
      ptx::tc_fence_after();
      const int m = mt * kBM + row;
      const int n0 = nt * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t v[16];
        ptx::tmem_ld_x16(lane_base + b * BN + 16 * c, v);
        ptx::tmem_wait_ld();
        if (m < M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + 16 * c + j;
            if (n < N) Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(__uint_as_float(v[j])));
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.acc_empty[b]);
      if (++b == C::kAccBufs) { b = 0; bph ^= 1; }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// X [N][K] fp16, box 64 (K) x BN (rows), 128-byte swizzle, zero fill past N.
cudaError_t make_x_map(CUtensorMap* map, const uint16_t* X, int N, int K, int BN) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int num_sms() {
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

template <int BN>
cudaError_t launch_bn(const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int N, cudaStream_t stream) {
  using C = Cfg<BN>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap map;
  cudaError_t e = make_x_map(&map, X, N, K, BN);
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(M, kBM) * ceil_div(N, BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_tc_kernel<BN><<<grid, kThreads, C::kSmemBytes, stream>>>(map, wq, s_p, z_p, Y, M, K, N);
  return cudaGetLastError();
}

}  // namespace

// The CUDA-core GEMV wins below this many tokens (measured N sweep, fused
// QKV shape); the tensor-core kernel from here on.
int gemv_max_n() { return 1; }

cudaError_t launch_gemm_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           const uint16_t* X, uint16_t* Y, int M, int K, int N, cudaStream_t stream) {
  if (K % kBK) return cudaErrorNotSupported;
  if (N <= 16) return launch_bn<16>(wq, scales, zeros, X, Y, M, K, N, stream);
  if (N <= 32) return launch_bn<32>(wq, scales, zeros, X, Y, M, K, N, stream);
  if (N <= 64) return launch_bn<64>(wq, scales, zeros, X, Y, M, K, N, stream);
  return launch_bn<128>(wq, scales, zeros, X, Y, M, K, N, stream);
}

namespace {

// One thread waits on an mbarrier whose phase nothing completes, with a short
// cycle budget: the wait must give up, record the timeout and return.
__global__ void wait_timeout_selftest_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
    wait_bar(&bar, 0, &abort_flag, &g_tc_status, true, limit);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(long long limit_cycles, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(limit_cycles);
  return cudaGetLastError();
}

cudaError_t read_and_clear_tc_status(int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_tc_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
}

}  // namespace w4a16
