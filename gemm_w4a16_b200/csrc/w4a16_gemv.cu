// Decode GEMV / few-token kernel (memory-bound regime).
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.3 item 2: the GEMV is memory
// bound; its design goals there are vectorised loads, unrolling to keep many
// loads in flight, the zero and scale of each int4 group at hand, the vector
// read through a fast on-chip path, and tiling both dimensions of the weight
// (rows and K) for parallelism.  On sm_100a:
//
//  * a CTA owns one 128-row block of the packed weight and a range of whole
//    groups along K; each of its 8 warps owns one 16-row tile of that block
//    and streams the tile's codes, scales and zeros straight from HBM into
//    registers with 16-byte non-allocating loads, 3 or 4 groups ahead of
//    the one it computes (no shared-memory staging, no barriers);
//  * the first groups are requested before the grid dependency wait, so with
//    programmatic dependent launch the weight stream starts while the
//    previous kernel finishes; the activations (written by that kernel) are
//    staged in shared memory after the wait;
//  * the products run on the tensor cores as warp-level mma.sync m16n8k16
//    (f16 inputs, fp32 accumulation): lane l = 4 g + c holds MMA rows g and
//    g + 8, which are the adjacent block rows 2 g and 2 g + 1 of the tile (so
//    one 32-bit load brings both scales and one byte both zero codes), and
//    chunk c (32 codes) of each; the exact dequant of one 32-bit word (8
//    codes) of each row gives the lane's A fragments of two MMAs, whose B
//    fragments are token g's activations at the same eight k (one 16-byte
//    shared load).  The MMA's k order is thus a permutation of the group that
//    A and B share; lanes of tokens g >= NT feed columns that are never
//    stored.  One MMA instruction replaces 256 fp32 FMAs, so the kernel issues
//    about 2.5 instructions per weight, 1.6 of them the exact dequant;
//  * split-K: CTAs of a thread-block cluster (up to 8 along K) reduce through
//    distributed shared memory into the cluster's rank-0 CTA in a fixed order
//    (deterministic, no atomics); the other ranks store their partial sums,
//    arrive on an mbarrier of rank 0 and leave at once, rank 0 waiting on it
//    (bounded).
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

#include <algorithm>

namespace w4a16 {

// Status word of the decode kernel's family: set when rank 0 of a cluster
// gives up waiting for the other ranks' partial sums (a bounded wait).
__device__ int g_gemv_status = 0;

namespace {

constexpr int kGvWarps = 8;                           // one 16-row MMA tile each
constexpr int kGvThreads = kGvWarps * 32;
// Groups of codes in flight per warp, in registers: 4 for one or two tokens
// (80 registers still hold them without spills; the decode step ran 1.255
// -> 1.224 ms, QKV at N = 2 9.7 -> 9.1 us with the 4-way row split), 3 with
// more tokens (4 was no faster at N = 4 and slower at N = 8) or the
// normalising prologue (which would spill).
template <int NT, bool kNorm>
__host__ __device__ constexpr int gv_depth() { return NT <= 2 && !kNorm ? 4 : NT > 8 ? 2 : 3; }
constexpr int kGvCtasPerSm = 3;                       // resident CTAs per SM (register budget)
constexpr int kGvWBytes = 4 * kRowBlock * 16;         // one group of 128 rows: 8 KB
constexpr int kMaxCluster = 8;
constexpr int kMaxXSmem = 64 * 1024;                  // largest staged activation slice
constexpr int kGvSmemLimit = 128 * 1024;              // dynamic shared memory a CTA may ask for
constexpr int kSmemPerSm = 228 * 1024;                // shared memory of one SM (sm_100)
constexpr int kSmemPerCta = 1024;                     // of it reserved per resident CTA
constexpr int kWideMaxM = 4096;                       // tallest weight given 16-token launches

// D += A B for one m16n8k16 tile: A 16 x 16 f16 (row), B 16 x 8 f16 (col),
// fp32 accumulators, in the warp-level fragment layout of mma.sync.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Non-allocating loads at p + OFF bytes (OFF folded into the instruction).
template <int OFF>
__device__ __forceinline__ uint4 ldg_v4_at(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "n"(OFF));
  return r;
}

// 16-byte asynchronous global -> shared copy (no register staging).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_addr(smem_dst)), "l"(src) : "memory");
}

template <int OFF>
__device__ __forceinline__ uint32_t ldg_u32_at(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1+%2];" : "=r"(v) : "l"(p), "n"(OFF));
  return v;
}

template <int OFF>
__device__ __forceinline__ uint32_t ldg_u8_at(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1+%2];" : "=r"(v) : "l"(p), "n"(OFF));
  return v;
}

// Halves between consecutive tokens of the staged activation slice: the
// slice of one token plus 16 halves, so the 16-byte loads of the two tokens
// in one quarter-warp fall on different banks.
__host__ __device__ inline int gv_xstride(int ng) { return ng * kGroup + 16; }

struct GvLayout {
  int x_off, red_off, cred_off, total;
};

__host__ __device__ inline GvLayout gv_layout(int nt, int gspan, int cl, int kw) {
  GvLayout L;
  L.x_off = 0;
  L.red_off = L.x_off + nt * gv_xstride(gspan) * 2;
  L.cred_off = L.red_off + kw * nt * kRowBlock * 4;
  L.total = L.cred_off + (cl > 1 ? cl * nt * kRowBlock * 4 : 0);
  return L;
}

// One group's operands of one lane: chunk c of the adjacent rows r (even)
// and r + 1 (two 16-byte halves of 32 contiguous bytes), their two scales
// (one 32-bit word) and the zero byte that holds both codes.
struct GvFrag {
  uint4 lo, hi;
  uint32_t s, z;
};

#ifdef W4A16_DEBUG_BOUNDS
// Index-check build: the extent of every buffer the CTA touches, set by
// thread 0 before any access.  A failed check records 2 in the status word
// (w4a16_device_status: W4A16_ERR_BOUNDS) and the access is skipped.
struct GvChk {
  const uint8_t *w0, *w1;     // packed codes
  const uint16_t *s0, *s1;    // packed scales
  const uint8_t *z0, *z1;     // packed zeros
  const uint16_t *x0, *x1;    // this launch's activations (global)
  const uint16_t *xs0, *xs1;  // the staged activation slice (shared)
  int red_n, cred_n;          // floats of the two partial-sum regions
};
__shared__ GvChk g_chk;

__device__ __forceinline__ bool gv_ok(bool ok) {
  if (!ok) atomicExch(&g_gemv_status, 2);
  return ok;
}
#endif

// Group J of the lane's streams: pw points at chunk c of row r of group 0,
// ps at the scale of row r, pz at the zero byte of rows r and r + 1.
template <int J>
__device__ __forceinline__ void gv_load(GvFrag& f, const uint8_t* pw, const uint16_t* ps, const uint8_t* pz) {
#ifdef W4A16_DEBUG_BOUNDS
  const uint8_t* w = pw + J * kGvWBytes;
  const uint16_t* sp = ps + J * kRowBlock;
  const uint8_t* zp = pz + J * (kRowBlock / 2);
  if (!gv_ok(w >= g_chk.w0 && w + 32 <= g_chk.w1 && sp >= g_chk.s0 && sp + 2 <= g_chk.s1 && zp >= g_chk.z0 &&
             zp + 1 <= g_chk.z1)) {
    f.lo = f.hi = make_uint4(0u, 0u, 0u, 0u);
    f.s = f.z = 0u;
    return;
  }
#endif
  f.lo = ldg_v4_at<J * kGvWBytes>(pw);
  f.hi = ldg_v4_at<J * kGvWBytes + 16>(pw);
  f.s = ldg_u32_at<J * kRowBlock * 2>(ps);
  f.z = ldg_u8_at<J * (kRowBlock / 2)>(pz);
}

template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "n"(SEL));
  return d;
}

// The dequant constants (as make_group_consts) of the lane's two rows at
// once: the two zero codes side by side in one register (row r in the low
// half), both fp16 forms built there, then each half copied to both halves.
__device__ __forceinline__ void gv_consts(const GvFrag& f, GroupConsts& lo, GroupConsts& hi) {
  const uint32_t t = f.z | (f.z << 12);                                   // code of row r + 1 at bits 16..19
  const uint32_t a = lop3_and_or(t, 0x000F000Fu, 0x64006400u);             // 1024 + z per half
  const uint32_t b = lop3_and_or(t << 4, 0x00F000F0u, 0xD400D400u);        // -(64 + z) per half
  lo.z1024 = prmt<0x1010>(a, a);
  hi.z1024 = prmt<0x3232>(a, a);
  lo.zneg64 = prmt<0x1010>(b, b);
  hi.zneg64 = prmt<0x3232>(b, b);
  lo.s2 = prmt<0x1010>(f.s, f.s);
  hi.s2 = prmt<0x3232>(f.s, f.s);
}

// The lane's accumulators: one m16n8 fragment per block of 8 tokens (NB = 2
// for 9 to 16 tokens, whose second block shares the dequantised A
// fragments), and the offset in halves of block j's activation row from
// block 0's.
template <int NB>
struct GvAcc {
  float c[NB][4];
  int xoff[NB];
};

// Dequantise one group of the lane's two rows and accumulate its eight MMAs
// per token block; xg points at token g's activations at k = 32 c of the
// group.
template <int NB>
__device__ __forceinline__ void gv_consume(const GvFrag& f, const uint16_t* xg, GvAcc<NB>& A) {
  GroupConsts clo, chi;
  gv_consts(f, clo, chi);
  const uint32_t wl[4] = {f.lo.x, f.lo.y, f.lo.z, f.lo.w};
  const uint32_t wh[4] = {f.hi.x, f.hi.y, f.hi.z, f.hi.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint4 xb[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const uint16_t* xp = xg + A.xoff[j] + 8 * t;
#ifdef W4A16_DEBUG_BOUNDS
      if (!gv_ok(xp >= g_chk.xs0 && xp + 8 <= g_chk.xs1)) xp = g_chk.xs0;
#endif
      xb[j] = *reinterpret_cast<const uint4*>(xp);
    }
    uint32_t al[4], ah[4];
    dequant_word(wl[t], clo, al);
    dequant_word(wh[t], chi, ah);
#pragma unroll
    for (int j = 0; j < NB; ++j) mma_16816(A.c[j], al[0], ah[0], al[1], ah[1], xb[j].x, xb[j].y);
#pragma unroll
    for (int j = 0; j < NB; ++j) mma_16816(A.c[j], al[2], ah[2], al[3], ah[3], xb[j].z, xb[j].w);
  }
}

template <int D, int U>
__device__ __forceinline__ void gv_load_first(GvFrag (&f)[D], int ng, const uint8_t* pw, const uint16_t* ps,
                                              const uint8_t* pz) {
  if constexpr (U < D) {
    if (U < ng) gv_load<U>(f[U], pw, ps, pz);
    gv_load_first<D, U + 1>(f, ng, pw, ps, pz);
  }
}

// Slots U.. of a step whose groups and refills all exist (no checks).
template <int D, int U, int NB>
__device__ __forceinline__ void gv_step_full(GvFrag (&f)[D], const uint8_t* pw, const uint16_t* ps,
                                             const uint8_t* pz, const uint16_t* xg, GvAcc<NB>& acc) {
  if constexpr (U < D) {
    gv_consume(f[U], xg + U * kGroup, acc);
    gv_load<U + D>(f[U], pw, ps, pz);
    gv_step_full<D, U + 1, NB>(f, pw, ps, pz, xg, acc);
  }
}

// Slots U.. of one step of D groups starting at group i0: consume group
// i0 + U from slot U, refill the slot with group i0 + U + D.
template <int D, int U, int NB>
__device__ __forceinline__ void gv_step(GvFrag (&f)[D], int i0, int ng, const uint8_t* pw,
                                        const uint16_t* ps, const uint8_t* pz, const uint16_t* xg,
                                        GvAcc<NB>& acc) {
  if constexpr (U < D) {
    if (i0 + U < ng) {
      gv_consume(f[U], xg + U * kGroup, acc);
      if (i0 + U + D < ng) gv_load<U + D>(f[U], pw, ps, pz);
      gv_step<D, U + 1, NB>(f, i0, ng, pw, ps, pz, xg, acc);
    }
  }
}

// The normalising prologue (w4a16_add_rmsnorm_gemm_qkv): X of the CTA's K
// range computed from the residual stream instead of read.  Each token row's
// sum of squares is formed over the whole row with exactly the thread
// mapping, chunk order and fixed-order reduction of add_rmsnorm_kernel (same
// thread count), so inv, X and r are bit-identical to that kernel's; then
// r = h + d, X = (r * inv) * gamma for the CTA's groups go to shared memory,
// and the CTAs of the first row block also write r for their K range.
template <int NT>
__device__ __forceinline__ void gv_norm_x(const NormIn& nin, int K, int ga, int ng, uint16_t* xs, int xstride,
                                          bool write_r) {
  static_assert(kGvThreads == kNormThreads, "the sum of squares must follow the norm kernel's order");
  __shared__ float wsum[kNormThreads / 32];
  __shared__ float s_inv[kGemvMaxTokens];
  const int chunks = K / 8;
#pragma unroll 1
  for (int n = 0; n < NT; ++n) {
    const uint4* hv = reinterpret_cast<const uint4*>(nin.h) + (size_t)n * chunks;
    const uint4* dv = nin.d ? reinterpret_cast<const uint4*>(nin.d) + (size_t)n * chunks : nullptr;
    // The norm kernel's per-thread order: chunks threadIdx.x, + 256, ...
    // (its batching of the loads does not change the order of the sum).
    float ss = 0.0f;
    for (int c = threadIdx.x; c < chunks; c += kNormThreads) {
      uint4 r = hv[c];
      if (dv) {
        const uint4 b = dv[c];
        r.x = hadd2_rn(r.x, b.x);
        r.y = hadd2_rn(r.y, b.y);
        r.z = hadd2_rn(r.z, b.z);
        r.w = hadd2_rn(r.w, b.w);
      }
      ss = sum_sq2(r.x, ss);
      ss = sum_sq2(r.y, ss);
      ss = sum_sq2(r.z, ss);
      ss = sum_sq2(r.w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      float tot = 0.0f;
#pragma unroll
      for (int w = 0; w < kNormThreads / 32; ++w) tot += wsum[w];
      s_inv[n] = rms_inv(tot, K, nin.eps);
    }
    __syncthreads();
  }
  const uint4* gv = reinterpret_cast<const uint4*>(nin.gamma);
  const int pieces = ng * (kGroup / 8);
  for (int idx = threadIdx.x; idx < NT * pieces; idx += kGvThreads) {
    const int n = idx / pieces, p = idx - n * pieces;
    const size_t c = (size_t)n * chunks + (size_t)ga * (kGroup / 8) + p;
    const uint4 a = reinterpret_cast<const uint4*>(nin.h)[c];
    uint4 r = a;
    if (nin.d) {
      const uint4 b = reinterpret_cast<const uint4*>(nin.d)[c];
      r.x = hadd2_rn(a.x, b.x);
      r.y = hadd2_rn(a.y, b.y);
      r.z = hadd2_rn(a.z, b.z);
      r.w = hadd2_rn(a.w, b.w);
    }
    if (write_r && nin.r_out) reinterpret_cast<uint4*>(nin.r_out)[c] = r;
    const uint4 g = gv[ga * (kGroup / 8) + p];
    const float inv = s_inv[n];
    uint4 o;
    o.x = scale2(r.x, g.x, inv);
    o.y = scale2(r.y, g.y, inv);
    o.z = scale2(r.z, g.z, inv);
    o.w = scale2(r.w, g.w, inv);
    *reinterpret_cast<uint4*>(xs + n * xstride + p * 8) = o;
  }
}

// KW = 1: the CTA's 8 warps are the 8 row tiles of a 128-row block; KW = 2
// or 4: 8 / KW row tiles (a half or a quarter of a block) with KW warps
// each, which take KW parts of the CTA's K range and meet in shared memory
// in a fixed order (more warps per row, and fewer or no cluster ranks, for
// shapes with few row blocks).  A CTA's rows stay whole 32-row groups, which
// the gate/up pairing needs.
template <int NT, int kEpi, int KW, bool kNorm>
__global__ void __launch_bounds__(kGvThreads, kGvCtasPerSm)
gemv_kernel(const uint8_t* __restrict__ wq, const uint16_t* __restrict__ s_p,
            const uint8_t* __restrict__ z_p, const uint16_t* __restrict__ X,
            uint16_t* __restrict__ Y, int M, int K, uint32_t cl_magic, int early, OutMap om, NormIn nin,
            int ntok) {
  extern __shared__ __align__(128) uint8_t smem[];
  // Tokens present: NT, or 9..NT for the two-block kernel (ntok).  X rows
  // past them are neither read nor staged and their outputs not stored.
  const int nt = NT > 8 ? ntok : NT;
  // Grid (row-block parts, cl): the cluster spans y, so blockIdx.y is the
  // CTA's rank along K and blockIdx.x its part of a row block; n / cl is
  // the high word of n * ceil(2^32 / cl) (exact for n < 2^32 / cl^2).
  const int cl = (int)gridDim.y;
  const int crank = (int)blockIdx.y;
  const int chunk = (int)blockIdx.x;
  auto div_cl = [&](int n) { return cl == 1 ? n : (int)__umulhi((uint32_t)n, cl_magic); };
  const int kg = K / kGroup;
  const int kc_n = K / kChunkK;
  const int gspan = div_cl(kg + cl - 1);
  const GvLayout L = gv_layout(NT, gspan, cl, KW);
  constexpr int kRows = kRowBlock / KW;    // rows of the CTA
  constexpr int kTiles = kGvWarps / KW;    // 16-row tiles of the CTA
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.x_off);  // [NT][xstride]
  float* red = reinterpret_cast<float*>(smem + L.red_off);     // [KW][NT][128]
  float* cred = reinterpret_cast<float*>(smem + L.cred_off);   // [cl][NT][128], rank 0 only

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int b = chunk / KW;
  const int ro = (chunk % KW) * kRows;     // the CTA's first row in the block
  const int ga = div_cl(kg * crank), gb = div_cl(kg * (crank + 1));
  const int ng = gb - ga;
  const int xstride = gv_xstride(ng);
  // This warp's tile and its share [gw0, gw0 + ngw) of the CTA's groups.
  const int tile = warp % kTiles, ks = warp / kTiles;
  const int gw0 = (ks * ng) / KW;
  const int ngw = ((ks + 1) * ng) / KW - gw0;

  ptx::griddep_launch_dependents();
#ifdef W4A16_DEBUG_BOUNDS
  if (threadIdx.x == 0) {
    const size_t blocks_all = (size_t)ceil_div(M, kRowBlock);
    g_chk.w0 = wq;
    g_chk.w1 = wq + blocks_all * kc_n * kRowBlock * 16;
    g_chk.s0 = s_p;
    g_chk.s1 = s_p + blocks_all * kg * kRowBlock;
    g_chk.z0 = z_p;
    g_chk.z1 = z_p + blocks_all * kg * (kRowBlock / 2);
    g_chk.x0 = X;
    g_chk.x1 = X ? X + (size_t)nt * K : X;
    const uint16_t* xs_base = reinterpret_cast<const uint16_t*>(smem + L.x_off);
    g_chk.xs0 = xs_base;
    g_chk.xs1 = xs_base + NT * xstride;
    g_chk.red_n = KW * NT * kRowBlock;
    g_chk.cred_n = cl > 1 ? cl * NT * kRowBlock : 0;
  }
  __syncthreads();
#endif
  __shared__ __align__(8) uint64_t s_done;
  if (cl > 1) {
    if (crank == 0 && threadIdx.x == 0) {
      ptx::mbar_init(&s_done, (uint32_t)((cl - 1) * kRows));
      ptx::fence_mbar_init();
    }
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  }

  // This lane's rows within the block: MMA rows g and g + 8 of the warp's
  // tile are the adjacent block rows rl and rl + 1.  Its group streams
  // (pointers at group ga; slot offsets are folded into the loads).
  const int rl = ro + 16 * tile + 2 * g;
  const int g0 = ga + gw0;
  const uint8_t* pw = wq + (size_t)b * kc_n * kRowBlock * 16 + (size_t)g0 * kGvWBytes + c * (kRowBlock * 16) + rl * 16;
  const uint16_t* ps = s_p + ((size_t)b * kg + g0) * kRowBlock + rl;
  const uint8_t* pz = z_p + ((size_t)b * kg + g0) * (kRowBlock / 2) + (rl >> 1);

  // The activations of this CTA's K range go to shared memory with
  // asynchronous 16-byte copies.  Without programmatic launch they are
  // requested first, so they do not queue behind the weight stream.
  auto stage_x = [&]() {
    const int pieces = ng * (kGroup / 8);
    if constexpr (NT == 1) {
      for (int p = threadIdx.x; p < pieces; p += kGvThreads) {
#ifdef W4A16_DEBUG_BOUNDS
        const uint16_t* src = X + (size_t)ga * kGroup + p * 8;
        if (!gv_ok(src >= g_chk.x0 && src + 8 <= g_chk.x1 && xs + p * 8 + 8 <= g_chk.xs1)) continue;
#endif
        cp_async16(xs + p * 8, X + (size_t)ga * kGroup + p * 8);
      }
    } else {
      for (int idx = threadIdx.x; idx < nt * pieces; idx += kGvThreads) {
        const int n = idx / pieces, p = idx - n * pieces;
#ifdef W4A16_DEBUG_BOUNDS
        const uint16_t* src = X + (size_t)n * K + (size_t)ga * kGroup + p * 8;
        if (!gv_ok(src >= g_chk.x0 && src + 8 <= g_chk.x1 && xs + n * xstride + p * 8 + 8 <= g_chk.xs1)) continue;
#endif
        cp_async16(xs + n * xstride + p * 8, X + (size_t)n * K + (size_t)ga * kGroup + p * 8);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (!early && !kNorm) stage_x();
  // The first groups depend on no earlier kernel: request them before the
  // grid dependency wait (which returns at once unless the launch is
  // programmatic); X (or the residual stream it comes from), written by that
  // kernel, only after it.
  constexpr int kDepth = gv_depth<NT, kNorm>();
  GvFrag f[kDepth];
  gv_load_first<kDepth, 0>(f, ngw, pw, ps, pz);
  ptx::griddep_wait();
  if constexpr (kNorm)
    gv_norm_x<NT>(nin, K, ga, ng, xs, xstride, chunk == 0);
  else if (early)
    stage_x();
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // Lane g's MMA column is token g of each block of 8; lanes of tokens
  // >= NT read token NT - 1: MMA columns are independent, and those columns
  // are never stored.
  constexpr int kNB = NT > 8 ? 2 : 1;
  GvAcc<kNB> acc;
#pragma unroll
  for (int j = 0; j < kNB; ++j) {
    acc.c[j][0] = acc.c[j][1] = acc.c[j][2] = acc.c[j][3] = 0.f;
    acc.xoff[j] = (min(8 * j + g, nt - 1) - min(g, nt - 1)) * xstride;
  }
  const uint16_t* xg = xs + min(g, nt - 1) * xstride + 32 * c + gw0 * kGroup;
  int i0 = 0;
  for (; i0 + 2 * kDepth <= ngw; i0 += kDepth) {   // every refill exists
    gv_step_full<kDepth, 0, kNB>(f, pw, ps, pz, xg, acc);
    pw += kDepth * kGvWBytes;
    ps += kDepth * kRowBlock;
    pz += kDepth * (kRowBlock / 2);
    xg += kDepth * kGroup;
  }
  for (; i0 < ngw; i0 += kDepth) {
    gv_step<kDepth, 0, kNB>(f, i0, ngw, pw, ps, pz, xg, acc);
    pw += kDepth * kGvWBytes;
    ps += kDepth * kRowBlock;
    pz += kDepth * (kRowBlock / 2);
    xg += kDepth * kGroup;
  }
  // Accumulator fragment j: MMA rows g (entries 0, 1: block row rl) and
  // g + 8 (entries 2, 3: block row rl + 1), tokens 8 j + 2 c and 8 j + 2 c + 1.
#pragma unroll
  for (int j = 0; j < kNB; ++j) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 8 * j + 2 * c + e;
      if (n < nt) {
#ifdef W4A16_DEBUG_BOUNDS
        if (!gv_ok((ks * NT + n) * kRowBlock + rl + 1 < g_chk.red_n)) continue;
#endif
        red[(ks * NT + n) * kRowBlock + rl] = acc.c[j][e];
        red[(ks * NT + n) * kRowBlock + rl + 1] = acc.c[j][2 + e];
      }
    }
  }
  __syncthreads();

  float tot[NT];
  const int rr = threadIdx.x;        // the CTA's rows: threads 0 .. kRows - 1
  const int r = ro + rr;             // row within the block
  // The fused form's destination and bias of row m, loaded before the
  // reductions so the load overlaps them.
  RowDst dst = {};
  if constexpr (kEpi == kEpiQkv) {
    const int m = b * kRowBlock + r;
    if (rr < kRows && crank == 0 && m < M) dst = row_dst(om, M, m);
  }
  if (rr < kRows) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sum = red[n * kRowBlock + r];
#pragma unroll
      for (int k = 1; k < KW; ++k) sum += red[(k * NT + n) * kRowBlock + r];   // K halves in order
      tot[n] = sum;
    }
  }

  if (cl > 1) {
    // Every CTA of the cluster has started once this wait returns, so rank
    // 0's shared memory and its arrival barrier may be used remotely.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (rr >= kRows) return;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#ifdef W4A16_DEBUG_BOUNDS
      if (!gv_ok((crank * NT + n) * kRowBlock + r < g_chk.cred_n)) continue;
#endif
      const uint32_t local = ptx::smem_addr(&cred[(crank * NT + n) * kRowBlock + r]);
      uint32_t remote;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(0));
      asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(remote), "f"(tot[n]) : "memory");
    }
    if (crank != 0) {
      // The other ranks announce their partial sums on rank 0's barrier
      // (release at cluster scope orders the stores above) and leave.
      uint32_t rbar;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(ptx::smem_addr(&s_done)), "r"(0));
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(rbar) : "memory");
      return;
    }
    // Rank 0: a bounded wait for every other rank's rows.
    {
      const long long t0 = clock64();
      while (true) {
        uint32_t ok;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0, 200000;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(ptx::smem_addr(&s_done)) : "memory");
        if (ok) break;
        if (clock64() - t0 > kWaitLimitCycles) {
          atomicExch(&g_gemv_status, 1);
          return;
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sum = 0.f;
      for (int c = 0; c < cl; ++c) sum += cred[(c * NT + n) * kRowBlock + r];
      tot[n] = sum;
    }
  } else if (rr >= kRows) {
    return;
  }

  const int m = b * kRowBlock + r;
  if constexpr (kEpi == kEpiGateUp) {
    // Threads 0 .. kRows - 1 are whole warps here: the gate/up pairing
    // shuffles within 32-row groups, which a CTA's rows never split.
#pragma unroll
    for (int n = 0; n < NT; ++n)
      if (n < nt) store_gate_up(om, b, r, n, tot[n], true);
  } else if (m < M) {
    if constexpr (kEpi == kEpiQkv) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        if (n < nt) store_row(dst, om.bias != nullptr, n, tot[n]);
    } else {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        if (n < nt) {
#ifdef W4A16_DEBUG_BOUNDS
          if (!gv_ok(m < M)) continue;
#endif
          Y[(size_t)n * M + m] = __half_as_ushort(__float2half_rn(tot[n]));
        }
    }
  }
}

template <int NT, int kEpi, int KW, bool kNorm = false>
cudaError_t launch_nt(const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int cl, bool pdl, cudaStream_t stream, const OutMap& om,
                      const NormIn& nin, int ntok) {
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemv_kernel<NT, kEpi, KW, kNorm>), kGvSmemLimit,
                                    smem_set);
  if (e != cudaSuccess) return e;
  const int blocks = ceil_div(M, kRowBlock);
  const GvLayout L = gv_layout(NT, ceil_div(K / kGroup, cl), cl, KW);
  if (L.total > kGvSmemLimit) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(blocks * KW), (unsigned)cl, 1);
  cfg.blockDim = dim3(kGvThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)cl;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  const uint32_t cl_magic = cl > 1 ? (uint32_t)((0x100000000ull + (unsigned)cl - 1) / (unsigned)cl) : 0u;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, kEpi, KW, kNorm>, wq, s_p, z_p, X, Y, M, K, cl_magic,
                            pdl ? 1 : 0, om, nin, ntok);
}

template <int kEpi, int KW, bool kNorm>
cudaError_t launch_kw(int nt, const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p, const uint16_t* X,
                      uint16_t* Y, int M, int K, int cl, bool pdl, cudaStream_t stream, const OutMap& om,
                      const NormIn& nin) {
  if constexpr (!kNorm)
    if (nt > 8) return launch_nt<16, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
  switch (nt) {
    case 1: return launch_nt<1, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 2: return launch_nt<2, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 3: return launch_nt<3, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 4: return launch_nt<4, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 5: return launch_nt<5, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 6: return launch_nt<6, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    case 7: return launch_nt<7, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
    default: return launch_nt<8, kEpi, KW, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, nt);
  }
}

// One launch of nt tokens (1..16; 9..16 as the 16-token kernel, whose extra
// columns repeat the last token) with row split kw (1, 2, or 4 at nt = 1).
template <int kEpi, bool kNorm = false>
cudaError_t launch_epi(int nt, int kw, const uint8_t* wq, const uint16_t* s_p, const uint8_t* z_p,
                       const uint16_t* X, uint16_t* Y, int M, int K, int cl, bool pdl, cudaStream_t stream,
                       const OutMap& om, const NormIn& nin) {
  if (kw == 4 && nt <= 2)   // the chooser takes KW = 4 for one or two tokens only
    return nt == 1 ? launch_nt<1, kEpi, 4, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, 1)
                   : launch_nt<2, kEpi, 4, kNorm>(wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin, 2);
  if (kw == 2) return launch_kw<kEpi, 2, kNorm>(nt, wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin);
  return launch_kw<kEpi, 1, kNorm>(nt, wq, s_p, z_p, X, Y, M, K, cl, pdl, stream, om, nin);
}

struct GvShape {
  int kw, cl;
};

}  // namespace

// Row split KW (1, 2 or 4 CTAs per 128-row block, see gemv_kernel) and cluster
// size along K (1..8), from the measured LLaMA N = 1 shapes.  First pass: all
// CTAs resident in one wave (kGvCtasPerSm per SM, set by the registers of one
// CTA), and at least 2.5 CTAs per SM on average when the shape allows it
// (fewer warps per SM hide the load and MMA latencies badly); among those
// the smallest busiest-SM work, ceil(CTAs / SMs) x the groups of one warp,
// then the larger KW (measured at equal CTA counts: gate/up 15.7 against
// 16.3 us, QKV 9.1 against 9.7 us with KW = 4 and no cluster), then the
// smaller cluster; when no choice reaches 2.5 CTAs per SM, the most CTAs.
// For one token, when that finds no dense single wave because the weight
// has too many row blocks for KW = 4 to fit in one wave, KW = 4 without a
// cluster over several waves instead (gate/up 22016 x 4096: 14.9 against
// 15.7 us; 28672 x 4096: 20.8 against 29.2 us; 128256 x 4096: 76.5 against
// 78.3 us; splitting such weights further along K was slower).  The staged
// activation slice must fit.
GvShape gemv_shape(int M, int K, int sms, int nt) {
  const int blocks = ceil_div(M, kRowBlock);
  const int kg = K / kGroup;
  const long long wave = (long long)kGvCtasPerSm * sms;
  GvShape best = {0, 0};
  long long best_key[4] = {0, 0, 0, 0};
  auto consider = [&](int kw, int cl, const long long (&key)[4]) {
    bool better = best.cl == 0;
    for (int i = 0; i < 4 && !better; ++i) {
      if (key[i] != best_key[i]) {
        better = key[i] < best_key[i];
        break;
      }
    }
    if (better) {
      best = {kw, cl};
      for (int i = 0; i < 4; ++i) best_key[i] = key[i];
    }
  };
  const int ntk = nt > 8 ? kGemvWideTokens : nt;   // tokens the launched kernel stages
  auto fits = [&](int kw, int cl) {
    return ntk * gv_xstride(ceil_div(kg, cl)) * 2 <= kMaxXSmem &&
           gv_layout(ntk, ceil_div(kg, cl), cl, kw).total <= kGvSmemLimit;
  };
  // CTAs one SM holds: the register budget, or fewer when the activation
  // slice and the partial sums fill its shared memory.
  auto wave_of = [&](int kw, int cl) {
    const int smem = gv_layout(ntk, ceil_div(kg, cl), cl, kw).total;
    return (long long)std::min(kGvCtasPerSm, kSmemPerSm / (smem + kSmemPerCta)) * sms;
  };
  auto load = [&](int kw, int cl) {
    const long long ctas = (long long)blocks * kw * cl;
    return (long long)ceil_div((int)ctas, sms) * ceil_div(ceil_div(kg, cl), kw);
  };
  // KW = 4 only for one or two tokens: at N = 4 it was no faster and at
  // N = 8 slower on every LLaMA-7B shape (down 17.4 against 11.9 us).
  for (int kw = 1; kw <= (nt <= 2 ? 4 : 2); kw *= 2) {
    for (int cl = 1; cl <= kMaxCluster && cl <= kg; ++cl) {
      if (!fits(kw, cl)) continue;
      const long long ctas = (long long)blocks * kw * cl;
      if ((kw > 1 || cl > 1) && ctas > wave_of(kw, cl)) continue;
      const bool dense = 2 * ctas >= 5LL * sms;
      const long long key[4] = {dense ? 0 : 1, dense ? load(kw, cl) : -ctas, -kw, cl};
      consider(kw, cl, key);
    }
  }
  const bool single_dense = best.cl > 0 && best_key[0] == 0 && (long long)blocks * best.kw * best.cl <= wave;
  if (nt == 1 && !single_dense && 4LL * blocks > wave && fits(4, 1)) return GvShape{4, 1};
  if (best.cl > 0) return best;
  // Nothing fits in one wave (many row blocks and a wide activation slice):
  // the smallest cluster whose slice fits, over several waves.
  for (int cl = 1; cl <= kMaxCluster && cl <= kg; ++cl)
    if (fits(1, cl)) return GvShape{1, cl};
  return GvShape{0, 0};   // no launch of this many tokens fits

}

cudaError_t launch_gemv(const uint8_t* wq, const uint16_t* scales, const uint8_t* zeros,
                        const uint16_t* X, uint16_t* Y, int M, int K, int N,
                        cudaStream_t stream, const OutMap* om, bool pdl, const NormIn* norm) {
  if (norm && (N > kGemvMaxTokens || !om || om->kind != kEpiQkv)) return cudaErrorNotSupported;
  const NormIn nin = norm ? *norm : NormIn{};
  // 9..16 tokens as one two-block launch on weights of up to kWideMaxM rows
  // (N = 9 / 16 on O 4096 x 4096: 8.2 / 8.5 against 11.3 / 12.5 us for
  // 8-token launches; taller weights ran slower that way: QKV 12288 x 4096
  // 17.9 against 17.4 us on the tile kernel, LLaMA-3 gate/up 28672 x 4096
  // 40.7 against 31.2 us); 8-token launches otherwise.
  const int per_launch = norm || M > kWideMaxM ? kGemvMaxTokens : kGemvWideTokens;
  for (int n0 = 0; n0 < N;) {
    int nt = std::min(per_launch, N - n0);
    GvShape sh = gemv_shape(M, K, num_sms(), nt);
    // A wide K leaves no room for 16 tokens' activations and partial sums in
    // one CTA: 8-token launches then.
    if (sh.cl == 0 && nt > kGemvMaxTokens) {
      nt = kGemvMaxTokens;
      sh = gemv_shape(M, K, num_sms(), nt);
    }
    if (sh.cl == 0) return cudaErrorNotSupported;
    const int ntk = nt > 8 ? kGemvWideTokens : nt;   // tokens the launched kernel stages
    const int cl = sh.cl;
    if (ntk * gv_xstride(ceil_div(K / kGroup, cl)) * 2 > kMaxXSmem) return cudaErrorNotSupported;
    const uint16_t* Xn = X ? X + (size_t)n0 * K : nullptr;
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
    if (norm)
      e = launch_epi<kEpiQkv, true>(nt, sh.kw, wq, scales, zeros, Xn, Yn, M, K, cl, pdl, stream, on, nin);
    else if (kind == kEpiGateUp)
      e = launch_epi<kEpiGateUp>(nt, sh.kw, wq, scales, zeros, Xn, Yn, M, K, cl, pdl, stream, on, nin);
    else if (kind == kEpiQkv)
      e = launch_epi<kEpiQkv>(nt, sh.kw, wq, scales, zeros, Xn, Yn, M, K, cl, pdl, stream, on, nin);
    else
      e = launch_epi<kEpiPlain>(nt, sh.kw, wq, scales, zeros, Xn, Yn, M, K, cl, pdl, stream, on, nin);
    if (e != cudaSuccess) return e;
    n0 += nt;
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
