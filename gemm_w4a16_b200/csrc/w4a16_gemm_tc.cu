// Large-N W4A16 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 1: with many tokens the
// GEMM is compute bound; it gets its own tiling, with the operands staged in
// shared memory to cut global traffic.  On sm_100a the tile is 128 weight
// rows x BN tokens, K walked in slots of 128 (one quantisation group):
//
//   warp 7 or 24  producer: X only (warp 7 when it is not an issuer).  One 3D TMA copy per X stage brings
//                 kXSlabs slabs of 64 k x BN tokens (128-byte swizzle, the
//                 K-major layout the MMA reads; rows past N and k past K are
//                 zero-filled).  Copies are 16-64 KB: on B200 an SM's bulk
//                 copy engine completes roughly one copy per several hundred
//                 cycles whatever its size, so few large copies are what
//                 keeps it ahead.
//   warps 8..23   dequantisers: four groups of four warps take the K slots in
//                 turn.  Thread = one weight row: it copies its row's 64
//                 bytes of codes (4 coalesced 16-byte cp.async, 512
//                 contiguous bytes per warp) and the group's scale and zero
//                 into its own kWDepth-deep shared-memory ring, so several
//                 slots per group are in flight without holding registers
//                 (each thread reads back only what it copied: no barrier);
//                 it dequantises exactly (dequant_word) and writes the fp16
//                 row slice into tensor memory with tcgen05.st: the MMA's A
//                 operand never touches shared memory.
//   warps 4..7    MMA issuers: 8 x tcgen05.mma kind::f16 (M = 128, N = BN,
//                 K = 16) per slot, A from TMEM, B = X from shared memory.
//                 On B200 one issuing thread completes a small-N MMA only
//                 every ~46 cycles, whatever N is below ~96, while the
//                 tensor core itself needs N / 2 cycles; so for BN <= 64 the
//                 K slots of a tile are dealt round-robin to kIssuers warps,
//                 each accumulating into its own fp32 TMEM tile (the
//                 epilogue adds them in a fixed order).  kIssuers divides
//                 both the number of A slots and its excess over the
//                 dequantiser groups, so no wait on an A-slot barrier can
//                 run two phases ahead (a parity wait cannot tell a phase
//                 from the one two steps later).  tcgen05.commit frees
//                 the A slot, the X stage (once every issuer is done with
//                 it) and, at the end of a tile, the accumulators.
//   warps 0..3    epilogue (and 24..27 at BN = 256, each of a lane quarter's
//                 two warps taking half of the columns): tcgen05.ld of the
//                 issuers' accumulators, their
//                 sum in issuer order, one RNE conversion to fp16, stores of
//                 Y[n][m].
//
// Persistent CTAs (one per SM) walk the tile list round-robin; the
// accumulator is double-buffered in TMEM when two fit next to the A slots.
// Every mbarrier wait is bounded: on expiry the kernel records a timeout in
// a device status word, stops issuing, drains its copies and MMAs, frees
// TMEM and returns.
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

namespace w4a16 {

__device__ int g_tc_status = 0;

namespace {

constexpr int kBM = 128;
constexpr int kMaxSlotK = 128;                   // k per TMEM A slot: 64 or 128
constexpr int kDqGroups = 4;                     // dequantiser groups (slots in flight)
constexpr int kFirstDqWarp = 8;
constexpr int kFirstIssuerWarp = 4;
constexpr int kLastDqWarp = kFirstDqWarp + 4 * kDqGroups - 1;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int BN>
struct Cfg {
  // k per TMEM A slot: half a quantisation group with few tokens (the
  // dequantiser groups then alternate between two slots each, see kASlots),
  // a whole group otherwise; fp16 pairs per 32-bit TMEM column.
  static constexpr int kSlotK = BN <= 128 ? 64 : 128;
  static constexpr int kAColsPerSlot = kSlotK / 2;
  static constexpr int kChunks = kSlotK / kChunkK;   // 16-byte chunks per row and slot
  static constexpr int kMmas = kSlotK / 16;          // K = 16 MMAs per slot
  // k per X stage: enough for a 16-64 KB copy, a multiple of 128.
  static constexpr int kXK = cmax(kMaxSlotK, cmin(512, (32768 / (BN * 2)) / kMaxSlotK * kMaxSlotK));
  static constexpr int kXSlabs = kXK / 64;
  static constexpr int kSlotsPerX = kXK / kSlotK;
  static constexpr int kXStageBytes = BN * kXK * 2;
  // Dequantiser rings: per group, kWDepth slots of 128 rows x (64 B codes,
  // 4 B scale pair, 4 B zero quad).
  // With many tokens (compute bound) one slot of prefetch in registers is
  // enough and the shared memory goes to the X ring instead.
  static constexpr bool kUseRing = BN <= 128;
  static constexpr int kWDepth = kUseRing ? 6 : 0;
  static constexpr int kWCodeBytes = kDqGroups * kWDepth * kRowBlock * kChunks * 16;
  static constexpr int kWMetaBytes = kDqGroups * kWDepth * kRowBlock * 4;
  static constexpr int kWRingBytes = kWCodeBytes + 2 * kWMetaBytes;
  static constexpr int kXStages = cmin(8, ((kUseRing ? 200 : 196) * 1024 - kWRingBytes) / kXStageBytes);
  // MMA issuer warps (one accumulator each) and accumulator buffers.
  // A slots in TMEM: with few tokens the MMA of a slot takes about as long
  // as its dequantisation, so twice as many slots as dequantiser groups let
  // each group fill one slot while the MMAs read its other one.
  static constexpr int kASlots = BN <= 128 ? 2 * kDqGroups : kDqGroups;
  static constexpr int kIssuers = BN <= 64 ? 4 : BN <= 128 ? 2 : 1;
  static constexpr int kAccCols = kIssuers * BN;
  static constexpr int kAccBufs = (2 * kAccCols + kASlots * kAColsPerSlot <= 512) ? 2 : 1;
  static constexpr int kACol0 = kAccBufs * kAccCols;
  static constexpr int kColsUsed = kACol0 + kASlots * kAColsPerSlot;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = ptx::idesc_f16_f32(kBM, BN);
  static constexpr int kBarBytes = 8 * (2 * kXStages + 2 * kASlots + 2 * kAccBufs + 1) + 16;
  static_assert(kACol0 + kASlots * kAColsPerSlot <= 512, "TMEM budget");
  static constexpr int kWOff = kXStages * kXStageBytes;
  static constexpr int kSmemUsed = kWOff + kWRingBytes + kBarBytes + 1024;
  // At least 120 KB so that one CTA owns an SM and all of its TMEM.
  static constexpr int kSmemBytes = kSmemUsed < 120 * 1024 ? 120 * 1024 : kSmemUsed;
  static_assert(kXStages >= 2, "X stage ring");
  static_assert(kIssuers >= 1 && kIssuers <= 4, "issuer warps are 4..7");
  // The X producer takes warp 7 when fewer than four issuers leave it free
  // (768 threads, more registers each), else a warp of its own after the
  // dequantisers.
  static constexpr int kProducerWarp = kIssuers < 4 ? kFirstIssuerWarp + 3 : kLastDqWarp + 1;
  // Epilogue warps: 0..3, plus 4 more after the others at BN = 256, where the
  // single accumulator keeps the tensor core idle while it is drained; each
  // epilogue warp of a TMEM lane quarter then drains half of the columns.
  static constexpr int kEpiWarps = BN == 256 ? 8 : 4;
  static constexpr int kBaseWarps = kIssuers < 4 ? kLastDqWarp + 1 : kLastDqWarp + 2;
  static constexpr int kThreads = (kBaseWarps + kEpiWarps - 4) * 32;
  // Parity waits see only the last phase's parity.  They stay exact when
  // every A slot has one consumer (kIssuers | kASlots) and the group
  // filling slot i, whose previous fill (slot i - kDqGroups) waited for the
  // use of slot i - kDqGroups - kASlots, thereby knows that slot
  // i - 2 kASlots is used too: both are the same issuer's, in order
  // (kIssuers | kASlots - kDqGroups).
  static_assert(kASlots % kIssuers == 0, "one consumer per A slot");
  static_assert(kASlots % kDqGroups == 0, "a group's slots step through the A slots in turn");
  static_assert((kASlots - kDqGroups) % kIssuers == 0, "in-order A-slot phases");
  static_assert(kXSlabs <= 8, "TMA box depth");
  static_assert(kColsUsed <= 512, "TMEM overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert((BN * 128) % 1024 == 0, "X slabs must stay 1024-byte aligned");
};

// Tile t -> (row tile mt, token tile nt).  Bands of kBand row tiles; inside
// a band the token tiles run fastest, so the CTAs working at the same time
// share a few weight blocks and every token tile of X in L2 instead of each
// holding its own weight block (valid for t < mt_n * nt_n).
constexpr int kBand = 8;

__device__ __forceinline__ void tile_coords(int t, int mt_n, int nt_n, int& mt, int& nt) {
  const int per_band = kBand * nt_n;
  const int band = t / per_band;
  const int rem = t - band * per_band;
  const int bm = cmin(kBand, mt_n - band * kBand);
  nt = rem / bm;
  mt = band * kBand + (rem - nt * bm);
}

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int BN, int kEpi>
__global__ void __launch_bounds__(Cfg<BN>::kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ wq,
               const uint16_t* __restrict__ s_p, const uint8_t* __restrict__ z_p,
               uint16_t* __restrict__ Y, int M, int K, int N, OutMap om) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kWOff + C::kWRingBytes);
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
  const int ks_n = K / C::kSlotK;                    // slots per tile
  const int nx = ceil_div(ks_n, C::kSlotsPerX);      // X stages per tile
  const int kc_n = K / kChunkK;
  const int kg = K / kGroup;
  const int my_tiles = (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kXStages; ++i) {
      ptx::mbar_init(&sh.x_full[i], 1);
      ptx::mbar_init(&sh.x_empty[i], C::kIssuers);   // every issuer, once per stage
    }
    for (int i = 0; i < C::kASlots; ++i) {
      ptx::mbar_init(&sh.a_full[i], 4);            // the 4 warps of one dequantiser group
      ptx::mbar_init(&sh.a_empty[i], 1);
    }
    for (int i = 0; i < C::kAccBufs; ++i) {
      ptx::mbar_init(&sh.acc_full[i], C::kIssuers);
      ptx::mbar_init(&sh.acc_empty[i], C::kEpiWarps);
    }
    ptx::mbar_init(sh.drain, C::kIssuers);
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

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int xs = 0;
      uint32_t xph = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, mt_n, nt_n, mt, nt);
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
  } else if (warp >= kFirstIssuerWarp && warp < kFirstIssuerWarp + C::kIssuers) {
    // --------------------------------------------------------- MMA issuers
    // Issuer ii takes the tile's slots ks = ii, ii + kIssuers, ...; A slot
    // and phase follow the CTA's running slot index, as the dequantisers
    // fill them.  Per X stage every issuer either commits (it read the
    // stage) or arrives (it had no slot there).
    const int ii = warp - kFirstIssuerWarp;
    if (lane == 0) {
      int xs = 0, b = 0;
      uint32_t xph = 0, bph = 0;
      bool ok = true;
      const uint64_t desc_x0 = ptx::smem_desc_sw128(ptx::smem_addr(smem));
      int tl = 0;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tl) {
        if (!wait_bar(&sh.acc_empty[b], bph ^ 1, sh.abort_flag, &g_tc_status)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * C::kAccCols + ii * BN;
        bool first = true;
        for (int xi = 0; ok && xi < nx; ++xi) {
          const int k0 = xi * C::kSlotsPerX;
          const int k1 = k0 + C::kSlotsPerX < ks_n ? k0 + C::kSlotsPerX : ks_n;
          bool used = false;
          for (int ks = k0 + ((ii - k0 % C::kIssuers) + C::kIssuers) % C::kIssuers; ks < k1;
               ks += C::kIssuers) {
            if (!used) {
              if (!wait_bar(&sh.x_full[xs], xph, sh.abort_flag, &g_tc_status)) { ok = false; break; }
              used = true;
            }
            const int sidx = tl * ks_n + ks;
            const int a = sidx % C::kASlots;
            const uint32_t aph = (uint32_t)((sidx / C::kASlots) & 1);
            if (!wait_bar(&sh.a_full[a], aph, sh.abort_flag, &g_tc_status)) { ok = false; break; }
            ptx::tc_fence_after();
            // B descriptor of the slot's first K = 16 step: the start-address
            // field (address / 16, low bits) moves with the offset in the ring.
            const uint64_t desc = desc_x0 + (uint64_t)((xs * C::kXStageBytes +
                                                        (ks - k0) * (C::kSlotK / 64) * (BN * 128)) >> 4);
            ptx::mma_ts_f16_slot<C::kMmas>(d_tmem, tmem + C::kACol0 + a * C::kAColsPerSlot, desc, C::kIdesc,
                                           first ? 0u : 1u, &sh.a_empty[a], (BN * 128) >> 4);
            first = false;
          }
          if (!ok) break;
          if (used) ptx::mma_commit(&sh.x_empty[xs]);
          else ptx::mbar_arrive(&sh.x_empty[xs]);
          if (++xs == C::kXStages) { xs = 0; xph ^= 1; }
        }
        if (!ok) break;
        ptx::mma_commit(&sh.acc_full[b]);
        if (++b == C::kAccBufs) { b = 0; bph ^= 1; }
      }
      // Drain: all MMAs issued by this thread have completed.
      ptx::mma_commit(sh.drain);
      wait_bar(sh.drain, 0, sh.abort_flag, &g_tc_status, false);
    }
  } else if (warp >= kFirstDqWarp && warp <= kLastDqWarp) {
    // -------------------------------------------------------- dequantisers
    // Group gi takes slots i = gi, gi + 4, ... of this CTA's sequence
    // (tile-major, then k), slot i lives in TMEM A slot i % kASlots.
    const int gi = (warp - kFirstDqWarp) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t a_lane = tmem + ((uint32_t)(quad * 32) << 16) + C::kACol0;
    const int n_slots = my_tiles * ks_n;
    // Refill cursor: the next slot to load, as (its index, its k slot g in
    // the tile, the tile's row block mt); advanced by kDqGroups slots at a
    // time without divisions.
    int f_i = gi, f_g = gi;
    int f_t = (int)blockIdx.x, f_mt = 0, f_nt = 0;
    while (f_g >= ks_n) { f_g -= ks_n; f_t += (int)gridDim.x; }
    if (f_t < tiles) tile_coords(f_t, mt_n, nt_n, f_mt, f_nt);
    auto advance = [&]() {
      f_i += kDqGroups;
      f_g += kDqGroups;
      bool moved = false;
      while (f_g >= ks_n) { f_g -= ks_n; f_t += (int)gridDim.x; moved = true; }
      if (moved && f_t < tiles) tile_coords(f_t, mt_n, nt_n, f_mt, f_nt);
    };
    int a = gi % C::kASlots;
    uint32_t aph = (uint32_t)((gi / C::kASlots) & 1);
    if constexpr (!C::kUseRing) {
      // Codes, scale and zero of the next slot in registers, one slot ahead.
      uint4 cur[C::kChunks], nxt[C::kChunks];
      uint32_t cur_s = 0, cur_z = 0, nxt_s = 0, nxt_z = 0;
      auto load = [&](uint4 (&v)[C::kChunks], uint32_t& sv, uint32_t& zv) {
        if (f_i < n_slots) {
          const int qg = f_g * C::kSlotK / kGroup;
          const uint4* src = reinterpret_cast<const uint4*>(wq) +
                             ((size_t)f_mt * kc_n + (size_t)f_g * C::kChunks) * kRowBlock + row;
#pragma unroll
          for (int j = 0; j < C::kChunks; ++j) v[j] = ldg_stream_v4(src + j * kRowBlock);
          sv = __ldg(s_p + ((size_t)f_mt * kg + qg) * kRowBlock + row);
          zv = (__ldg(z_p + ((size_t)f_mt * kg + qg) * (kRowBlock / 2) + (row >> 1)) >> ((row & 1) * 4)) & 0xFu;
        }
        advance();
      };
      load(cur, cur_s, cur_z);
      for (int i = gi; i < n_slots; i += kDqGroups) {
        load(nxt, nxt_s, nxt_z);
        const GroupConsts gc = make_group_consts(cur_z, (uint16_t)cur_s);
        if (!wait_bar_warp(&sh.a_empty[a], aph ^ 1, sh.abort_flag, &g_tc_status)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int hlf = 0; hlf < C::kChunks / 2; ++hlf) {
          // 16 columns at a time: with the next slot's codes held in
          // registers, a 32-column buffer would not fit the thread's share.
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t h[16];
            const uint4 w = cur[hlf * 2 + c];
            dequant_word(w.x, gc, &h[0]);
            dequant_word(w.y, gc, &h[4]);
            dequant_word(w.z, gc, &h[8]);
            dequant_word(w.w, gc, &h[12]);
            ptx::tmem_st_x16(a_lane + a * C::kAColsPerSlot + hlf * 32 + c * 16, h);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.a_full[a]);
        a += kDqGroups;
        if (a >= C::kASlots) { a -= C::kASlots; aph ^= 1; }
#pragma unroll
        for (int j = 0; j < C::kChunks; ++j) cur[j] = nxt[j];
        cur_s = nxt_s;
        cur_z = nxt_z;
      }
    } else {
      // This thread's ring: codes [gi][stage][chunk j][row] x 16 B, then the
      // scale pair and zero quad words [gi][stage][row] x 4 B.
      const uint32_t ring = ptx::smem_addr(smem + C::kWOff);
      auto code_at = [&](int st, int j) {
        return ring + (uint32_t)((((gi * C::kWDepth + st) * C::kChunks + j) * kRowBlock + row) * 16);
      };
      auto s_at = [&](int st) {
        return ring + (uint32_t)(C::kWCodeBytes + ((gi * C::kWDepth + st) * kRowBlock + row) * 4);
      };
      auto z_at = [&](int st) { return s_at(st) + (uint32_t)C::kWMetaBytes; };
      // Copy the cursor's slot (if it exists) into stage st and advance the
      // cursor; always closes a cp.async group, so that "all but the newest
      // kWDepth - 1 groups" means "the oldest slot in the ring is in".
      auto issue = [&](int st) {
        if (f_i < n_slots) {
          const int qg = f_g * C::kSlotK / kGroup;        // quantisation group of the slot
          const uint4* src = reinterpret_cast<const uint4*>(wq) +
                             ((size_t)f_mt * kc_n + (size_t)f_g * C::kChunks) * kRowBlock + row;
#pragma unroll
          for (int j = 0; j < C::kChunks; ++j) cp_async16(code_at(st, j), src + j * kRowBlock);
          // 4-byte words holding this row's scale (rows row & ~1, row | 1) and
          // zero nibble (rows (row & ~7) .. (row | 7)).
          cp_async4(s_at(st), s_p + ((size_t)f_mt * kg + qg) * kRowBlock + (row & ~1));
          cp_async4(z_at(st), z_p + ((size_t)f_mt * kg + qg) * (kRowBlock / 2) + ((row >> 1) & ~3));
        }
        cp_async_commit();
        advance();
      };
#pragma unroll
      for (int d = 0; d < C::kWDepth; ++d) issue(d);
      int st = 0;
      for (int i = gi; i < n_slots; i += kDqGroups) {
        cp_async_wait<C::kWDepth - 1>();
        uint4 v[C::kChunks];
#pragma unroll
        for (int j = 0; j < C::kChunks; ++j) v[j] = ptx::lds_v4(code_at(st, j));
        const uint32_t sw = ptx::lds_u32(s_at(st));
        const uint32_t zw = ptx::lds_u32(z_at(st));
        const uint16_t sv = (uint16_t)(sw >> ((row & 1) * 16));
        const uint32_t zv = (zw >> (((row >> 1) & 3) * 8 + (row & 1) * 4)) & 0xFu;
        const GroupConsts gc = make_group_consts(zv, sv);
        if (!wait_bar_warp(&sh.a_empty[a], aph ^ 1, sh.abort_flag, &g_tc_status)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int hlf = 0; hlf < C::kChunks / 2; ++hlf) {
          uint32_t h[32];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 w = v[hlf * 2 + c];
            dequant_word(w.x, gc, &h[c * 16 + 0]);
            dequant_word(w.y, gc, &h[c * 16 + 4]);
            dequant_word(w.z, gc, &h[c * 16 + 8]);
            dequant_word(w.w, gc, &h[c * 16 + 12]);
          }
          ptx::tmem_st_x32(a_lane + a * C::kAColsPerSlot + hlf * 32, h);
        }
        // The stage's contents are consumed (the dequantised values depend on
        // them); refill it with this group's slot kWDepth turns ahead.
        issue(st);
        if (++st == C::kWDepth) st = 0;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.a_full[a]);
        a += kDqGroups;
        if (a >= C::kASlots) { a -= C::kASlots; aph ^= 1; }
      }
      // Nothing may still be writing this CTA's shared memory at exit.
      cp_async_wait<0>();
    }
  } else if (warp < 4 || warp >= C::kBaseWarps) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    // Columns of this warp: all, or one half when two warps share a quarter.
    constexpr int kCols = BN * 4 / C::kEpiWarps;
    const int col0 = warp < 4 ? 0 : kCols;
    int b = 0;
    uint32_t bph = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, mt_n, nt_n, mt, nt);
      const int m = mt * kBM + row;
      const int n0 = nt * BN + col0;
      // The fused form's destination and bias of this row, loaded before the
      // wait so the load overlaps it.
      RowDst dst = {};
      if constexpr (kEpi == kEpiQkv) {
        if (m < M) dst = row_dst(om, M, m);
      }
      if (!wait_bar_warp(&sh.acc_full[b], bph, sh.abort_flag, &g_tc_status)) break;
      ptx::tc_fence_after();
      // Issuers that own no slot of this tile (K < kIssuers slots) wrote nothing.
      const int parts = ks_n < C::kIssuers ? ks_n : C::kIssuers;
      // Drain the accumulator 16 columns at a time, software-pipelined: the
      // issuer-0 part of chunk c + 1 is in flight while chunk c is converted
      // and stored; the buffer is handed back to the MMA issuers as soon as
      // its last columns are in registers.
      const uint32_t acc0 = lane_base + b * C::kAccCols + col0;
      uint32_t nxt[16];
      ptx::tmem_ld_x16(acc0, nxt);
#pragma unroll 1
      for (int c = 0; c < kCols / 16; ++c) {
        ptx::tmem_wait_ld();
        float sum[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) sum[j] = __uint_as_float(nxt[j]);
        if (c + 1 < kCols / 16) ptx::tmem_ld_x16(acc0 + 16 * (c + 1), nxt);
        for (int p = 1; p < parts; ++p) {
          uint32_t v[16];
          ptx::tmem_ld_x16(acc0 + p * BN + 16 * c, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) sum[j] += __uint_as_float(v[j]);
        }
        if (c + 1 == kCols / 16) {
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.acc_empty[b]);
        }
        if constexpr (kEpi == kEpiGateUp) {
          // Whole warps, two tokens at a time with every lane busy: a gate
          // lane hands g(n + 1) to its up partner (lane ^ 16) and takes u(n)
          // in one exchange, then writes H[n]; the up lane writes H[n + 1].
          // Per output the arithmetic is store_gate_up's (the same bits); the
          // lane's H pointer steps two token rows per pair.
          const bool up = (row & 16) != 0;
          const int i = gate_up_channel(mt, row & ~16);
          const int nb = n0 + 16 * c + (up ? 1 : 0);
          uint16_t* hp = om.h + (size_t)nb * om.mi + i;
          const size_t step = 2 * (size_t)om.mi;
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float recv = __shfl_xor_sync(0xffffffffu, up ? sum[j] : sum[j + 1], 16);
            const float g = up ? recv : sum[j];
            const float u = up ? sum[j + 1] : recv;
            if (nb + j < N && i < om.mi) {
              const float silu = __fdividef(g, 1.0f + __expf(-g));
              *hp = __half_as_ushort(__float2half_rn(silu * u));
            }
            hp += step;
          }
        } else if (m < M) {
          if constexpr (kEpi == kEpiQkv) {
            // The row's destination pointer steps by its pitch from token to
            // token (store_row's arithmetic, without a 64-bit multiply per
            // element).
            const int nb = n0 + 16 * c;
            uint16_t* p = dst.y + (size_t)nb * dst.ld;
            const bool has_bias = om.bias != nullptr;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (nb + j < N) {
                float v = sum[j];
                if (has_bias) v = __fadd_rn(v, dst.bias);
                *p = __half_as_ushort(__float2half_rn(v));
              }
              p += dst.ld;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = n0 + 16 * c + j;
              if (n < N) Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(sum[j]));
            }
          }
        }
      }
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

template <int BN, int kEpi>
cudaError_t launch_bn(const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int N, cudaStream_t stream, const OutMap& om) {
  using C = Cfg<BN>;
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemm_tc_kernel<BN, kEpi>), C::kSmemBytes,
                                    smem_set);
  if (e != cudaSuccess) return e;
  CUtensorMap map;
  e = make_x_map(&map, X, N, K, BN, C::kXSlabs);
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(M, kBM) * ceil_div(N, BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_tc_kernel<BN, kEpi><<<grid, C::kThreads, C::kSmemBytes, stream>>>(map, wq, s_p, z_p, Y, M, K, N, om);
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

// The decode kernel runs up to this many tokens (one launch; measured N sweep,
// fused QKV shape); the tensor-core tile kernel from there on.
int gemv_max_n() { return kGemvMaxTokens; }

template <int kEpi>
cudaError_t launch_tc_map(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros, const uint16_t* X,
                          uint16_t* Y, int M, int K, int N, cudaStream_t stream, const OutMap& om) {
  if (N <= 16) return launch_bn<16, kEpi>(wq, scales, zeros, X, Y, M, K, N, stream, om);
  if (N <= 32) return launch_bn<32, kEpi>(wq, scales, zeros, X, Y, M, K, N, stream, om);
  if (N <= 64) return launch_bn<64, kEpi>(wq, scales, zeros, X, Y, M, K, N, stream, om);
  if (N <= 128) return launch_bn<128, kEpi>(wq, scales, zeros, X, Y, M, K, N, stream, om);
  return launch_bn<256, kEpi>(wq, scales, zeros, X, Y, M, K, N, stream, om);
}

cudaError_t launch_gemm_tc(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                           const uint16_t* X, uint16_t* Y, int M, int K, int N, cudaStream_t stream,
                           const OutMap* om) {
  if (K % kMaxSlotK) return cudaErrorNotSupported;
  if (om && om->kind == kEpiGateUp)
    return launch_tc_map<kEpiGateUp>(wq, scales, zeros, X, nullptr, M, K, N, stream, *om);
  if (om) return launch_tc_map<kEpiQkv>(wq, scales, zeros, X, nullptr, M, K, N, stream, *om);
  return launch_tc_map<kEpiPlain>(wq, scales, zeros, X, Y, M, K, N, stream, OutMap{});
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
