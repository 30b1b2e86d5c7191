// Decode GEMV / few-token product on the tensor cores, with the weight
// stream split evenly over every SM (sm_100a).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 2: with one token (or a
// few) the product is a GEMV, bound by memory; the goal is to keep the weight
// stream at memory speed and hide the arithmetic, tiling the weight along
// both its rows and K so that every compute unit has a share.  On sm_100a:
//
//  * Unit = (128-row block b, quantisation group g): 8 KB of codes, 256 B of
//    scales and 64 B of zeros, each contiguous in its packed array, units in
//    block-major order.  CTA c of G takes units [c U / G, (c + 1) U / G) of
//    the U = blocks x groups units, so every SM streams the same bytes for
//    any M and K (a block may be split between consecutive CTAs).
//  * One producer thread copies each unit (three bulk copies) and its
//    activation tile (one TMA copy of BN tokens x 128 k, 128-byte swizzle,
//    the K-major layout the MMA reads; tokens past N zero-filled) into a
//    ring of shared-memory stages.
//  * Dequantiser groups of four warps (thread = weight row) take the units in
//    turn: exact in-register dequant (dequant_word), tcgen05.st of the row's
//    128 fp16 weights into a TMEM A slot.  Issuer warps take the units in
//    turn and run eight tcgen05.mma kind::f16 (M = 128, N = BN, K = 16) from
//    the A slot and the X tile into their own fp32 accumulator in TMEM (one
//    issuing thread completes a small-N MMA only every few tens of cycles,
//    so several issue side by side).
//  * Epilogue warps (one per TMEM lane quarter): at the end of each of the
//    CTA's blocks, tcgen05.ld of the issuers' accumulators, summed in issuer
//    order.  A block the CTA covers entirely is rounded once to fp16 and
//    written.  Otherwise the fp32 partial goes to the caller's workspace; the
//    last CTA to finish the block's lane quarter (an atomic counter per block
//    and quarter) adds the partials of all of the block's CTAs in CTA order,
//    rounds once and writes Y, then resets the counter.  Deterministic, no
//    floating-point atomics, and no CTA ever waits for another.
//  * Footprint: about 100 KB of shared memory, 256 TMEM columns and at most
//    32 K registers, so two CTAs fit on an SM.  With programmatic dependent
//    launch the next call's CTAs then start streaming their weights while
//    this call's CTAs finish; X, Y and the workspace are touched only after
//    the grid dependency wait.
//  * Every mbarrier wait is bounded: on expiry the kernel records a timeout
//    in a device status word, stops, drains its copies and MMAs, frees TMEM
//    and returns.
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

namespace w4a16 {

__device__ int g_gvtc_status = 0;

namespace {

constexpr int kUnitCodes = kRowBlock * kGroup / 2;    // 8192 B of codes per unit
constexpr int kUnitS = kRowBlock * 2;                 // 256 B of scales
constexpr int kUnitZ = kRowBlock / 2;                 // 64 B of zeros
constexpr int kUnitW = kUnitCodes + kUnitS + kUnitZ;  // one weight stage
constexpr int kHalfK = kGroup / 2;                    // k per A slot: half a unit
constexpr int kACols = kHalfK / 2;                    // TMEM columns of one A slot (fp16 pairs)

template <int BN_, int XROWS, int DQ, int ACCB, int WSTAGES, int XSTAGES>
struct GtCfg {
  static constexpr int BN = BN_;            // MMA N
  // Token rows an activation tile holds: BN, or 8 when at most 8 tokens are
  // real (the MMA's rows 8..15 then read the next 1 KB of shared memory,
  // which only reaches accumulator columns that are never read).
  static constexpr int kXRows = XROWS;
  static constexpr int kDq = DQ;            // dequantiser groups of four warps
  static constexpr int kIss = DQ;           // MMA issuer warps, one accumulator each
  // TMEM A slots of half a unit (64 k): two per group, so the MMAs of one
  // half run while the group dequantises the other.
  static constexpr int kASlots = 2 * DQ;
  static constexpr int kAccBufs = ACCB;     // accumulator sets
  // Two rings: weight stages of kDq consecutive units (one per dequantiser
  // group; freed once every group has read its codes into registers),
  // filled by the producer warp with three copies per stage (codes, scales,
  // zeros) issued from three lanes at once; and one-unit activation tiles
  // (freed by the MMAs' commit), filled by each issuer for its own units a
  // few units ahead.  The weight stream is never held back by MMA latency,
  // and a copy of the codes moves kDq x 8 KB.
  static constexpr int kWStages = WSTAGES;
  static constexpr int kStageBytes = DQ * kUnitW;
  static constexpr int kXStages = XSTAGES;
  static constexpr int kXAhead = XSTAGES / DQ;     // activation tiles in flight per issuer
  static constexpr int kSlab = kXRows * 128;       // one 64-k slab of a tile
  static constexpr int kXBytes = 2 * kSlab;
  static constexpr int kAccCols = kIss * BN;
  static constexpr int kACol0 = kAccBufs * kAccCols;
  static constexpr int kTmemCols = 256;
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kRowBlock, BN);
  // Warps: 0..3 epilogue, 4..4+kIss-1 issuers, then the weight producer,
  // then the dequantiser groups.
  static constexpr int kFirstIss = 4;
  static constexpr int kWProducer = kFirstIss + kIss;
  static constexpr int kFirstDq = kWProducer + 1;
  static constexpr int kThreads = (kFirstDq + 4 * kDq) * 32;
  // Shared memory: X ring (1024-byte aligned tiles), weight ring, barriers.
  static constexpr int kXOff = 0;
  static constexpr int kWOff = kXStages * kXBytes;
  static constexpr int kBarOff = kWOff + kWStages * kStageBytes;
  static constexpr int kNumBars = 2 * kWStages + 2 * kXStages + 2 * kASlots + 2 * kAccBufs + 1;
  static constexpr int kSmemBytes = kBarOff + 8 * kNumBars + 16 + 1024;

  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 64, "MMA N");
  static_assert(kACol0 + kASlots * kACols <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");
  static_assert(kXBytes % 1024 == 0, "swizzled X tiles stay 1024-byte aligned");
  static_assert(kXRows == BN || (kXRows == 8 && BN == 16), "activation tile rows");
  static_assert(kXAhead >= 1, "activation tiles in flight");
  // A parity wait cannot tell a phase from the one two steps later.  The
  // waits below stay exact because each waiter saw the barrier's previous
  // phase: every group waits on every phase of every weight stage; unit i
  // belongs to group and issuer i mod kDq, its halves to A slots
  // 2 (i mod kDq) and 2 (i mod kDq) + 1, and its activation stage
  // i mod kXStages is used by that issuer only (kDq divides kXStages).
  static_assert(kXStages % kDq == 0, "activation ring");
};

// Units [start(c), start(c + 1)) belong to CTA c.
__host__ __device__ __forceinline__ long long unit_start(long long U, int G, int c) {
  return U * c / G;
}

// The CTA whose range holds unit u.
__host__ __device__ __forceinline__ int cta_of(long long U, int G, long long u) {
  return (int)(((u + 1) * G - 1) / U);
}

template <class C, int kEpi>
__global__ void __launch_bounds__(C::kThreads, 2)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ wq,
               const uint16_t* __restrict__ s_p, const uint8_t* __restrict__ z_p, uint16_t* __restrict__ Y,
               int M, int K, int N, uint32_t* __restrict__ ws_cnt, float* __restrict__ ws_part, OutMap om) {
  constexpr int BN = C::BN;
  constexpr int SW = C::kWStages;
  constexpr int SX = C::kXStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* wfull = bars;
  uint64_t* wempty = wfull + SW;
  uint64_t* xfull = wempty + SW;
  uint64_t* xempty = xfull + SX;
  uint64_t* a_full = xempty + SX;
  uint64_t* a_empty = a_full + C::kASlots;
  uint64_t* acc_full = a_empty + C::kASlots;
  uint64_t* acc_empty = acc_full + C::kAccBufs;
  uint64_t* drain = acc_empty + C::kAccBufs;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kg = K / kGroup;
  const int nb = ceil_div(M, kRowBlock);
  const long long U = (long long)nb * kg;
  const int G = (int)gridDim.x;
  const int c = (int)blockIdx.x;
  const int u0 = (int)unit_start(U, G, c);
  const int u1 = (int)unit_start(U, G, c + 1);
  const int L = u1 - u0;                      // units of this CTA (>= 1: G <= U)
  const int b_first = u0 / kg;
  const int nblk = (u1 - 1) / kg - b_first + 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SW; ++i) {
      ptx::mbar_init(&wfull[i], 1);
      ptx::mbar_init(&wempty[i], 4 * C::kDq);  // the 4 warps of every group
    }
    for (int i = 0; i < SX; ++i) {
      ptx::mbar_init(&xfull[i], 1);
      ptx::mbar_init(&xempty[i], 1);          // the unit's issuer, by commit
    }
    for (int i = 0; i < C::kASlots; ++i) {
      ptx::mbar_init(&a_full[i], 4);
      ptx::mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < C::kAccBufs; ++i) {
      ptx::mbar_init(&acc_full[i], C::kIss);
      ptx::mbar_init(&acc_empty[i], 4);
    }
    ptx::mbar_init(drain, C::kIss);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == C::kFirstIss) {
    ptx::tmem_alloc(tmem_ptr, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  ptx::griddep_launch_dependents();
  const uint32_t tmem = *tmem_ptr;

  if (warp == C::kWProducer) {
    // ----------------------------------------------------- weight producer
    // The weights do not depend on the kernels before this one in the
    // stream, so this warp never waits for them.  Stage t holds units
    // t kDq .. t kDq + kDq - 1 (fewer at the CTA's end): their codes,
    // scales and zeros are each one contiguous range, copied by lanes 0, 1
    // and 2 in the same instruction.
    const int n_st = (L + C::kDq - 1) / C::kDq;
    int issued = 0;
    for (int t = 0; t < n_st; ++t) {
      if (t >= SW && !wait_bar_warp(&wempty[t % SW], (uint32_t)(((t / SW) & 1) ^ 1), abort_flag, &g_gvtc_status))
        break;
      const int i = t * C::kDq;
      const int nu = L - i < C::kDq ? L - i : C::kDq;
      uint8_t* dst = smem + C::kWOff + (t % SW) * C::kStageBytes;
      uint64_t* bar = &wfull[t % SW];
      if (lane == 0) ptx::mbar_arrive_expect_tx(bar, (uint32_t)(nu * kUnitW));
      __syncwarp();
      if (lane == 0)
        ptx::bulk_load(dst, wq + (size_t)(u0 + i) * kUnitCodes, (uint32_t)(nu * kUnitCodes), bar);
      else if (lane == 1)
        ptx::bulk_load(dst + C::kDq * kUnitCodes, reinterpret_cast<const uint8_t*>(s_p) + (size_t)(u0 + i) * kUnitS,
                       (uint32_t)(nu * kUnitS), bar);
      else if (lane == 2)
        ptx::bulk_load(dst + C::kDq * (kUnitCodes + kUnitS), z_p + (size_t)(u0 + i) * kUnitZ,
                       (uint32_t)(nu * kUnitZ), bar);
      issued = t + 1;
    }
    // Drain: every copy issued into this CTA's shared memory has landed.
    for (int t = issued - SW > 0 ? issued - SW : 0; t < issued; ++t)
      wait_bar(&wfull[t % SW], (uint32_t)((t / SW) & 1), abort_flag, &g_gvtc_status, false);
  } else if (warp >= C::kFirstIss && warp < C::kFirstIss + C::kIss) {
    // --------------------------------------------------------- MMA issuers
    // Issuer ii takes the CTA's units i = ii, ii + kIss, ...; per block it
    // accumulates its units into its own BN columns of the block's
    // accumulator set, and arrives (commit, or a plain arrive when it had
    // no unit there) on the set's "full" barrier.
    const int ii = warp - C::kFirstIss;
    if (lane == 0) {
      const uint64_t desc0 = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kXOff));
      // This issuer's units i = ii + k kIss, k < n_my; unit i's activation
      // tile lives in X stage i mod kXStages, a stage only this issuer uses.
      const int n_my = ii < L ? (L - ii + C::kIss - 1) / C::kIss : 0;
      auto issue_x = [&](int i) {
        uint64_t* bar = &xfull[i % SX];
        ptx::mbar_arrive_expect_tx(bar, C::kXBytes);
        ptx::tma_load_3d(smem + C::kXOff + (i % SX) * C::kXBytes, &tmap_x, bar, 0, 0, 2 * ((u0 + i) % kg));
      };
      // X may be written by the kernel before this one: only after the grid
      // dependency wait.
      ptx::griddep_wait();
      int x_issued = 0;
      for (; x_issued < C::kXAhead && x_issued < n_my; ++x_issued) issue_x(ii + x_issued * C::kIss);
      bool ok = true;
      int cur = -1;              // block being accumulated (CTA-local index)
      bool first = true;         // no MMA of this issuer in block `cur` yet
      // Close block `cur` (arrive on its "full" barrier: commit if this issuer
      // issued MMAs there) and open the next one once the epilogue has freed
      // its accumulator set.
      auto next_block = [&]() -> bool {
        if (cur >= 0) {
          uint64_t* f = &acc_full[cur % C::kAccBufs];
          if (first) ptx::mbar_arrive(f);
          else ptx::mma_commit(f);
        }
        ++cur;
        first = true;
        if (!wait_bar(&acc_empty[cur % C::kAccBufs], (uint32_t)(((cur / C::kAccBufs) & 1) ^ 1), abort_flag,
                      &g_gvtc_status))
          return false;
        ptx::tc_fence_after();
        return true;
      };
      for (int k = 0; ok && k < n_my; ++k) {
        const int i = ii + k * C::kIss;
        const int bl = (u0 + i) / kg - b_first;
        while (ok && cur < bl) ok = next_block();
        if (!ok) break;
        // Refill the stage of this issuer's previous unit once its MMAs are done.
        if (k >= 1 && x_issued < n_my) {
          const int ip = i - C::kIss;
          if (!wait_bar(&xempty[ip % SX], (uint32_t)((ip / SX) & 1), abort_flag, &g_gvtc_status)) break;
          issue_x(ii + x_issued * C::kIss);
          ++x_issued;
        }
        const int st = i % SX;
        if (!wait_bar(&xfull[st], (uint32_t)((i / SX) & 1), abort_flag, &g_gvtc_status)) break;
        const uint32_t d_tmem = tmem + (cur % C::kAccBufs) * C::kAccCols + ii * BN;
        // The unit's two halves: four K = 16 MMAs each, over the matching
        // 64-k slab of the activation tile.
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int j = 2 * i + hf;
          const int a = j % C::kASlots;
          if (!wait_bar(&a_full[a], (uint32_t)((j / C::kASlots) & 1), abort_flag, &g_gvtc_status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t desc = desc0 + (uint64_t)((st * C::kXBytes + hf * C::kSlab) >> 4);
          ptx::mma_ts_f16_slot<4>(d_tmem, tmem + C::kACol0 + a * kACols, desc, C::kIdesc,
                                  (first && hf == 0) ? 0u : 1u, &a_empty[a], 0u);
        }
        if (!ok) break;
        ptx::mma_commit(&xempty[st]);
        first = false;
      }
      // Every block of the CTA gets this issuer's arrival, units or not.
      while (ok && cur < nblk - 1) ok = next_block();
      if (ok && cur >= 0) {
        uint64_t* f = &acc_full[cur % C::kAccBufs];
        if (first) ptx::mbar_arrive(f);
        else ptx::mma_commit(f);
      }
      // Drain: all MMAs issued by this thread have completed, and every
      // activation copy it issued has landed.
      ptx::mma_commit(drain);
      wait_bar(drain, 0, abort_flag, &g_gvtc_status, false);
      for (int k = 0; k < x_issued; ++k) {
        const int i = ii + k * C::kIss;
        if (k + C::kXAhead >= x_issued)
          wait_bar(&xfull[i % SX], (uint32_t)((i / SX) & 1), abort_flag, &g_gvtc_status, false);
      }
    }
  } else if (warp >= C::kFirstDq) {
    // -------------------------------------------------------- dequantisers
    // Group gi takes units i = gi, gi + kDq, ...; thread = row of the block.
    const int gi = (warp - C::kFirstDq) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t a_lane = tmem + ((uint32_t)(quad * 32) << 16) + C::kACol0;
    const uint32_t wring = ptx::smem_addr(smem + C::kWOff);
    for (int i = gi; i < L; i += C::kDq) {
      // Unit i is unit gi of weight stage t = i / kDq.
      const int t = i / C::kDq;
      const int st = t % SW;
      if (!wait_bar_warp(&wfull[st], (uint32_t)((t / SW) & 1), abort_flag, &g_gvtc_status)) break;
      const uint32_t sbase = wring + st * C::kStageBytes;
      const uint32_t base = sbase + gi * kUnitCodes;
      const uint4 v0 = ptx::lds_v4(base + 0 * 2048 + row * 16);
      const uint4 v1 = ptx::lds_v4(base + 1 * 2048 + row * 16);
      const uint4 v2 = ptx::lds_v4(base + 2 * 2048 + row * 16);
      const uint4 v3 = ptx::lds_v4(base + 3 * 2048 + row * 16);
      const uint32_t sv = ptx::lds_u16(sbase + C::kDq * kUnitCodes + gi * kUnitS + row * 2);
      const uint32_t zb = ptx::lds_u8(sbase + C::kDq * (kUnitCodes + kUnitS) + gi * kUnitZ + (row >> 1));
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&wempty[st]);
      const GroupConsts gc = make_group_consts((zb >> ((row & 1) * 4)) & 0xFu, (uint16_t)sv);
      bool ok = true;
      // Two halves of 64 k, each into its own A slot: chunks (v0, v1), then (v2, v3).
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int j = 2 * i + hf;
        const int a = j % C::kASlots;
        const uint32_t dst = a_lane + a * kACols;
        const uint4 c0 = hf ? v2 : v0, c1 = hf ? v3 : v1;
        uint32_t h[16];
        dequant_word(c0.x, gc, &h[0]);
        dequant_word(c0.y, gc, &h[4]);
        dequant_word(c0.z, gc, &h[8]);
        dequant_word(c0.w, gc, &h[12]);
        if (!wait_bar_warp(&a_empty[a], (uint32_t)(((j / C::kASlots) & 1) ^ 1), abort_flag, &g_gvtc_status)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::tmem_st_x16(dst, h);
        dequant_word(c1.x, gc, &h[0]);
        dequant_word(c1.y, gc, &h[4]);
        dequant_word(c1.z, gc, &h[8]);
        dequant_word(c1.w, gc, &h[12]);
        ptx::tmem_st_x16(dst + 16, h);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&a_full[a]);
      }
      if (!ok) break;
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    // Outputs and the workspace may still be in use by the kernel before
    // this one until the grid dependency is resolved.
    ptx::griddep_wait();
    for (int bi = 0; bi < nblk; ++bi) {
      const int b = b_first + bi;
      const int i0 = (b * kg > u0 ? b * kg : u0) - u0;
      const int i1 = ((b + 1) * kg < u1 ? (b + 1) * kg : u1) - u0;
      const int span = i1 - i0;
      const int buf = bi % C::kAccBufs;
      const int m = b * kRowBlock + row;
      RowDst rd = {};
      if constexpr (kEpi == kEpiQkv) {
        if (m < M) rd = row_dst(om, M, m);
      }
      // Tokens 8 h .. 8 h + 7 of row m: rounded once and written (whole
      // warps call this: the gate/up pairing shuffles).
      auto store8 = [&](int h, const float (&v)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = h * 8 + j;
          if constexpr (kEpi == kEpiGateUp) {
            store_gate_up(om, b, row, n, v[j], n < N);
          } else if (n < N && m < M) {
            if constexpr (kEpi == kEpiQkv) store_row(rd, om.bias != nullptr, n, v[j]);
            else Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(v[j]));
          }
        }
      };
      if (!wait_bar_warp(&acc_full[buf], (uint32_t)((bi / C::kAccBufs) & 1), abort_flag, &g_gvtc_status)) break;
      ptx::tc_fence_after();
      const bool whole = span == kg;
      // A split block's fp32 share goes to this CTA's workspace slot (0 for
      // the CTA's first block, 1 for its last).
      float* part = ws_part + (size_t)(c * 2 + (bi == 0 ? 0 : 1)) * N * kRowBlock + row;
      // Eight tokens at a time, up to the last real one: the issuers'
      // accumulators in issuer order.
      const int chunks = ((N < BN ? N : BN) + 7) / 8;
#pragma unroll 1
      for (int h = 0; h < chunks; ++h) {
        float v[8];
        bool have = false;
#pragma unroll
        for (int p = 0; p < C::kIss; ++p) {
          // Issuer p owns a unit of this block iff one of i0 .. i1 - 1 is p mod kIss.
          if (span < C::kIss && ((p - i0 % C::kIss) + C::kIss) % C::kIss >= span) continue;
          uint32_t t[8];
          ptx::tmem_ld_x8(lane_base + buf * C::kAccCols + p * BN + h * 8, t);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = have ? v[j] + __uint_as_float(t[j]) : __uint_as_float(t[j]);
          have = true;
        }
        if (whole) {
          store8(h, v);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (h * 8 + j < N) part[(size_t)(h * 8 + j) * kRowBlock] = v[j];
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);

      if (!whole) {
        // The last of the block's CTAs (per lane quarter) adds every CTA's
        // partial in CTA order and writes the row.
        ptx::fence_acq_rel_gpu();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = ptx::atom_add_acq_rel_gpu(&ws_cnt[b * 4 + quad], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        const int cf = cta_of(U, G, (long long)b * kg);
        const int cl = cta_of(U, G, (long long)(b + 1) * kg - 1);
        if (old == (uint32_t)(cl - cf)) {
          ptx::fence_acq_rel_gpu();
#pragma unroll 1
          for (int h = 0; h < chunks; ++h) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0.f;
            for (int cc = cf; cc <= cl; ++cc) {
              const int sl = (long long)b == unit_start(U, G, cc) / kg ? 0 : 1;
              const float* pp = ws_part + (size_t)(cc * 2 + sl) * N * kRowBlock + row;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (h * 8 + j < N) v[j] += __ldcg(pp + (size_t)(h * 8 + j) * kRowBlock);
            }
            store8(h, v);
          }
          if (lane == 0) ws_cnt[b * 4 + quad] = 0u;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kFirstIss) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Up to 8 tokens: three dequantiser groups (and issuers), one accumulator
// set, three weight stages of three units (24.9 KB) and nine activation
// stages of 8 token rows (2 KB), three per issuer.
using Cfg8 = GtCfg<16, 8, 3, 1, 3, 9>;
// Up to 16 tokens: as above with 16-row activation tiles (4 KB), two per issuer.
using Cfg16 = GtCfg<16, 16, 3, 1, 3, 6>;
// Up to 32 tokens: two groups, two accumulator sets, four weight stages of
// two units (16.6 KB) and four activation stages (8 KB).
using Cfg32 = GtCfg<32, 32, 2, 2, 4, 4>;
// Up to 64 tokens: two groups, one accumulator set, two weight stages of
// two units and four activation stages (16 KB).
using Cfg64 = GtCfg<64, 64, 2, 1, 2, 4>;

int grid_for(int M, int K) {
  const long long U = (long long)ceil_div(M, kRowBlock) * (K / kGroup);
  const int sms = num_sms();
  return (int)(U < sms ? U : sms);
}

template <class C, int kEpi>
cudaError_t launch_cfg(const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                       uint16_t* Y, int M, int K, int N, void* ws, bool pdl, cudaStream_t stream,
                       const OutMap& om) {
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemv_tc_kernel<C, kEpi>), C::kSmemBytes,
                                    smem_set);
  if (e != cudaSuccess) return e;
  CUtensorMap map;
  e = make_x_map(&map, X, N, K, C::kXRows, 2);
  if (e != cudaSuccess) return e;
  uint32_t* cnt = static_cast<uint32_t*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + gemv_tc_counter_bytes(M));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_for(M, K), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_tc_kernel<C, kEpi>, map, wq, s_p, z_p, Y, M, K, N, cnt, part, om);
}

}  // namespace

size_t gemv_tc_counter_bytes(int M) {
  return ((size_t)ceil_div(M, kRowBlock) * 4 * sizeof(uint32_t) + 255) / 256 * 256;
}

size_t gemv_tc_workspace_bytes(int M, int K, int N) {
  return gemv_tc_counter_bytes(M) + (size_t)grid_for(M, K) * 2 * N * kRowBlock * sizeof(float);
}

cudaError_t launch_gemv_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros, const uint16_t* X,
                           uint16_t* Y, int M, int K, int N, void* workspace, bool pdl, cudaStream_t stream,
                           const OutMap* om) {
  if (N > kGemvTcMaxTokens) return cudaErrorNotSupported;
  // The split-block counters must start at zero.  A completed call leaves
  // its own counters at zero, but a call with more row blocks reaches bytes
  // that an earlier, smaller call used for its fp32 partials: clear them.
  cudaError_t e = cudaMemsetAsync(workspace, 0, gemv_tc_counter_bytes(M), stream);
  if (e != cudaSuccess) return e;
  const int kind = om ? om->kind : kEpiPlain;
  const OutMap o = om ? *om : OutMap{};
  uint16_t* y = om ? nullptr : Y;
#define W4A16_GVTC(CFG)                                                                               \
  do {                                                                                                \
    if (kind == kEpiGateUp) return launch_cfg<CFG, kEpiGateUp>(wq, scales, zeros, X, y, M, K, N,      \
                                                                workspace, pdl, stream, o);           \
    if (kind == kEpiQkv) return launch_cfg<CFG, kEpiQkv>(wq, scales, zeros, X, y, M, K, N, workspace, \
                                                         pdl, stream, o);                             \
    return launch_cfg<CFG, kEpiPlain>(wq, scales, zeros, X, y, M, K, N, workspace, pdl, stream, o);   \
  } while (0)
  if (N <= 8) W4A16_GVTC(Cfg8);
  if (N <= 16) W4A16_GVTC(Cfg16);
  if (N <= 32) W4A16_GVTC(Cfg32);
  W4A16_GVTC(Cfg64);
#undef W4A16_GVTC
}

// ------------------------------------------------ allocation-free variant
//
// Scratch of w4a16_gemm_noalloc: the split-block counters and fp32 partials
// of the split decode kernel live in this fixed device array instead of a
// caller workspace, so that call allocates nothing.  Every GPU that loads the
// library holds the array until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];

// Device address of the array on the current device, looked up once per
// device (the first call on a device does it, with that device current).
cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *ptr = p;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_gemv_tc_noalloc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                                   const uint16_t* X, uint16_t* Y, int M, int K, int N, bool pdl,
                                   cudaStream_t stream) {
  if (N > kGemvTcMaxTokens || gemv_tc_workspace_bytes(M, K, N) > kNoallocScratchBytes)
    return cudaErrorNotSupported;
  void* ws = nullptr;
  const cudaError_t e = noalloc_scratch(&ws);
  if (e != cudaSuccess) return e;
  // launch_gemv_tc clears the counters first; the partials are written
  // before they are read.
  return launch_gemv_tc(wq, scales, zeros, X, Y, M, K, N, ws, pdl, stream, nullptr);
}

cudaError_t read_and_clear_gvtc_status(int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_gvtc_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_gvtc_status, &zero, sizeof(int));
}

}  // namespace w4a16
