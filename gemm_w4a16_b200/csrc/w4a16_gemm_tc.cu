// Large-N W4A16 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1: with many tokens the
// GEMM is compute bound; it gets its own tiling, with the operands staged in
// shared memory to cut global traffic.  On sm_100a the tile is 128 weight
// rows x BN tokens, K walked in slots of 128 (one quantisation group):
//
//   warp 4        producer: X only.  One 3D TMA copy per X stage brings
//                 kXSlabs slabs of 64 k x BN tokens (128-byte swizzle, the
//                 K-major layout the MMA reads; rows past N and k past K are
//                 zero-filled).  Copies are 16-64 KB: on B200 an SM's bulk
//                 copy engine completes roughly one copy per several hundred
//                 cycles whatever its size, so few large copies are what
//                 keeps it ahead.
//   warps 8..23   dequantisers: four groups of four warps take the K slots in
//                 turn.  Thread = one weight row: it loads its row's 64 bytes
//                 of codes (4 coalesced 16-byte loads, 512 contiguous bytes
//                 per warp) and the group's scale and zero straight from
//                 global memory, one slot ahead, dequantises exactly
//                 (dequant_word) and writes the fp16 row slice into tensor
//                 memory with tcgen05.st: the MMA's A operand never touches
//                 shared memory.
//   warp 5        MMA issuer: 8 x tcgen05.mma kind::f16 (M = 128, N = BN,
//                 K = 16) per slot, A from TMEM, B = X from shared memory,
//                 fp32 accumulator in TMEM; tcgen05.commit frees the A slot,
//                 the X stage and, at the end of a tile, the accumulator.
//   warps 0..3    epilogue: tcgen05.ld of the accumulator, one RNE
//                 conversion to fp16, stores of Y[n][m].
//
// Persistent CTAs (one per SM) walk the tile list round-robin; the
// accumulator is double-buffered in TMEM when two fit next to the A slots.
// Every mbarrier wait is bounded: on expiry the kernel records a timeout in
// a device status word, stops issuing, drains its copies and MMAs, frees
// TMEM and returns.
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace w4a16 {

__device__ int g_tc_status = 0;

namespace {

constexpr int kBM = 128;
constexpr int kSlotK = 128;                      // k per TMEM A slot (one group)
constexpr int kAColsPerSlot = kSlotK / 2;        // fp16 pairs per 32-bit column
constexpr int kDqGroups = 4;                     // dequantiser groups (slots in flight)
constexpr int kFirstDqWarp = 8;
constexpr int kThreads = (kFirstDqWarp + 4 * kDqGroups) * 32;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int BN>
struct Cfg {
  // k per X stage: enough for a 16-64 KB copy, a multiple of the slot size.
  static constexpr int kXK = cmax(kSlotK, cmin(512, (32768 / (BN * 2)) / kSlotK * kSlotK));
  static constexpr int kXSlabs = kXK / 64;
  static constexpr int kSlotsPerX = kXK / kSlotK;
  static constexpr int kXStageBytes = BN * kXK * 2;
  static constexpr int kXStages = cmin(8, (196 * 1024) / kXStageBytes);
  static constexpr int kAccBufs = (2 * BN + kDqGroups * kAColsPerSlot <= 512) ? 2 : 1;
  static constexpr int kACol0 = kAccBufs * BN;
  static constexpr int kASlots = kDqGroups;
  static constexpr int kColsUsed = kACol0 + kASlots * kAColsPerSlot;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kBM, BN);
  static constexpr int kBarBytes = 8 * (2 * kXStages + 2 * kASlots + 2 * kAccBufs + 1) + 16;
  static constexpr int kSmemUsed = kXStages * kXStageBytes + kBarBytes + 1024;
  // At least 120 KB so that one CTA owns an SM and all of its TMEM.
  static constexpr int kSmemBytes = kSmemUsed < 120 * 1024 ? 120 * 1024 : kSmemUsed;
  static_assert(kXStages >= 2, "X stage ring");
  static_assert(kXSlabs <= 8, "TMA box depth");
  static_assert(kColsUsed <= 512, "TMEM overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert((BN * 128) % 1024 == 0, "X slabs must stay 1024-byte aligned");
};

struct Shared {
  uint64_t* x_full;
  uint64_t* x_empty;
  uint64_t* a_full;
  uint64_t* a_empty;
  uint64_t* acc_full;
  uint64_t* acc_empty;
  uint64_t* drain;
  uint32_t* tmem_ptr;
  volatile int* abort_flag;
};

// Codes of one 128-k slot for one row (four 16-byte chunks) plus the group's
// scale and zero, held in registers between the load and the dequantisation.
struct SlotRegs {
  uint4 v[4];
  uint16_t s;
  uint32_t z;
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kXStages * C::kXStageBytes);
  Shared sh;
  sh.x_full = bars;
  sh.x_empty = sh.x_full + C::kXStages;
  sh.a_full = sh.x_empty + C::kXStages;
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
  const int ks_n = K / kSlotK;                       // slots per tile
  const int nx = ceil_div(ks_n, C::kSlotsPerX);      // X stages per tile
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;
  const int my_tiles = (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kXStages; ++i) {
      ptx::mbar_init(&sh.x_full[i], 1);
      ptx::mbar_init(&sh.x_empty[i], 1);
    }
    for (int i = 0; i < C::kASlots; ++i) {
      ptx::mbar_init(&sh.a_full[i], 4);            // the 4 warps of one dequantiser group
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
      int xs = 0;
      uint32_t xph = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int nt = t / mt_n;
        for (int xi = 0; xi < nx; ++xi) {
          if (!wait_bar(&sh.x_empty[xs], xph ^ 1, sh.abort_flag, &g_tc_status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&sh.x_full[xs], C::kXStageBytes);
          ptx::tma_load_3d(smem + xs * C::kXStageBytes, &tmap_x, &sh.x_full[xs], 0, nt * BN,
                           xi * C::kXSlabs);
          issued_mask |= 1u << xs;
          issued_par = (issued_par & ~(1u << xs)) | (xph << xs);
          if (++xs == C::kXStages) { xs = 0; xph ^= 1; }
        }
      }
      // Drain: every copy issued into this CTA's shared memory has landed.
      for (int i = 0; i < C::kXStages; ++i)
        if (issued_mask & (1u << i))
          wait_bar(&sh.x_full[i], (issued_par >> i) & 1u, sh.abort_flag, &g_tc_status, false);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int xs = 0, a = 0, b = 0;
      uint32_t xph = 0, aph = 0, bph = 0;
      bool ok = true;
      const uint32_t x_base = ptx::smem_addr(smem);
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        if (!wait_bar(&sh.acc_empty[b], bph ^ 1, sh.abort_flag, &g_tc_status)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * BN;
        for (int ks = 0; ks < ks_n; ++ks) {
          const int sub = ks % C::kSlotsPerX;
          if (sub == 0 && !wait_bar(&sh.x_full[xs], xph, sh.abort_flag, &g_tc_status)) { ok = false; break; }
          if (!wait_bar(&sh.a_full[a], aph, sh.abort_flag, &g_tc_status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t xslab = x_base + xs * C::kXStageBytes + sub * 2 * (BN * 128);
          const uint32_t acol = tmem + C::kACol0 + a * kAColsPerSlot;
          uint32_t a_cols[8];
          uint64_t b_desc[8];
#pragma unroll
          for (int j = 0; j < kSlotK / 16; ++j) {
            a_cols[j] = acol + 8 * j;
            b_desc[j] = ptx::smem_desc_sw128(xslab + (j >> 2) * (BN * 128) + (j & 3) * 32);
          }
          ptx::mma_ts_f16_x8(d_tmem, a_cols, b_desc, C::kIdesc, ks != 0);
          ptx::mma_commit(&sh.a_empty[a]);
          if (++a == C::kASlots) { a = 0; aph ^= 1; }
          if (sub == C::kSlotsPerX - 1 || ks == ks_n - 1) {
            ptx::mma_commit(&sh.x_empty[xs]);
            if (++xs == C::kXStages) { xs = 0; xph ^= 1; }
          }
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
    // Group gi takes slots i = gi, gi + 4, ... of this CTA's sequence
    // (tile-major, then k), slot i lives in TMEM A slot i % kASlots.
    const int gi = (warp - kFirstDqWarp) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t a_lane = tmem + ((uint32_t)(quad * 32) << 16) + C::kACol0;
    const long long n_slots = (long long)my_tiles * ks_n;
    auto load_slot = [&](long long i, SlotRegs& r) {
      const int tl = (int)(i / ks_n);
      const int g = (int)(i - (long long)tl * ks_n);
      const int mt = (blockIdx.x + tl * gridDim.x) % mt_n;
      const uint4* src = reinterpret_cast<const uint4*>(wq) + ((size_t)mt * kc_n + (size_t)g * 4) * kRowBlock + row;
#pragma unroll
      for (int j = 0; j < 4; ++j) r.v[j] = ldg_stream_v4(src + j * kRowBlock);
      r.s = __ldg(s_p + ((size_t)mt * kg + g) * kRowBlock + row);
      r.z = __ldg(z_p + ((size_t)mt * kg + g) * (kRowBlock / 2) + (row >> 1));
    };
    SlotRegs cur, nxt;
    if (gi < n_slots) load_slot(gi, cur);
    for (long long i = gi; i < n_slots; i += kDqGroups) {
      if (i + kDqGroups < n_slots) load_slot(i + kDqGroups, nxt);
      const int a = (int)(i % C::kASlots);
      const uint32_t aph = (uint32_t)((i / C::kASlots) & 1);
      const GroupConsts gc = make_group_consts((cur.z >> ((row & 1) * 4)) & 0xFu, cur.s);
      if (!wait_bar_warp(&sh.a_empty[a], aph ^ 1, sh.abort_flag, &g_tc_status)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint32_t h[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 v = cur.v[hlf * 2 + c];
          dequant_word(v.x, gc, &h[c * 16 + 0]);
          dequant_word(v.y, gc, &h[c * 16 + 4]);
          dequant_word(v.z, gc, &h[c * 16 + 8]);
          dequant_word(v.w, gc, &h[c * 16 + 12]);
        }
        ptx::tmem_st_x32(a_lane + a * kAColsPerSlot + hlf * 32, h);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.a_full[a]);
      cur = nxt;
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

// X [N][K] fp16 viewed as a 3D tensor (64 k, N rows, K/64 slabs): the box
// (64, BN, slabs) lands as `slabs` K-major 128-byte-swizzled tiles of BN x 64,
// the layout the MMA's B descriptor describes.  Zero fill past N and K.
cudaError_t make_x_map(CUtensorMap* map, const uint16_t* X, int N, int K, int BN, int slabs) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)(K / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)BN, (cuuint32_t)slabs};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(X), dims, strides, box,
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
  cudaError_t e = make_x_map(&map, X, N, K, BN, C::kXSlabs);
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(M, kBM) * ceil_div(N, BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_tc_kernel<BN><<<grid, kThreads, C::kSmemBytes, stream>>>(map, wq, s_p, z_p, Y, M, K, N);
  return cudaGetLastError();
}

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

// The CUDA-core GEMV runs up to this many tokens (measured N sweep, fused QKV
// shape); the tensor-core kernel from there on.
int gemv_max_n() { return 4; }

cudaError_t launch_gemm_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           const uint16_t* X, uint16_t* Y, int M, int K, int N, cudaStream_t stream) {
  if (K % kSlotK) return cudaErrorNotSupported;
  if (N <= 16) return launch_bn<16>(wq, scales, zeros, X, Y, M, K, N, stream);
  if (N <= 32) return launch_bn<32>(wq, scales, zeros, X, Y, M, K, N, stream);
  if (N <= 64) return launch_bn<64>(wq, scales, zeros, X, Y, M, K, N, stream);
  if (N <= 128) return launch_bn<128>(wq, scales, zeros, X, Y, M, K, N, stream);
  return launch_bn<256>(wq, scales, zeros, X, Y, M, K, N, stream);
}

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
