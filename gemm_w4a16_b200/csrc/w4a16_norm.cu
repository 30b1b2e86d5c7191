// Residual add + RMS normalisation, the operator that produces the
// projections' input X.
//
// "PerfXLLM on Snapdragon 8 Gen2", section 3.2, first fusion: the residual
// connection's addition and the normalisation run as one operator, so the sum
// reaches the normalisation without a trip through global memory.  The page
// names the two operations only; per token row, the reading taken is
//
//   r = fp16_RN(h + d)                   (one f16x2 add; d absent: r = h)
//   X = fp16_RN((r * inv) * gamma),      inv = 1 / sqrt(mean(r^2) + eps),
//
// the mean of squares, the root and the products in fp32, X rounded once.
//
// One CTA per token row.  Pass 1 loads up to four 16-byte chunks of h and d
// per thread before storing anything, forms r, keeps it in shared memory
// (and writes it out when asked) and sums its squares; a fixed-order block
// reduction gives the mean; pass 2 scales r from shared memory.  h and d are
// read once and r and X written once: 8 bytes of HBM traffic per channel plus
// gamma, which stays in L2 across rows.  Bound by HBM.
//
// The kernel lets the next kernel in the stream be scheduled as soon as it
// starts (programmatic dependent launch): a projection launched with early
// weight streaming then reads its weights while this runs, and reads X only
// after this kernel has completed.
#include "w4a16_internal.cuh"
#include "sm100_ptx.cuh"

namespace w4a16 {

namespace {


// h, d and r_out may be the same memory as each other (r_out == h or d: each
// element is read before the same thread writes it); X overlaps none of them.
__global__ void __launch_bounds__(kNormThreads)
add_rmsnorm_kernel(const uint16_t* h, const uint16_t* d, const uint16_t* __restrict__ gamma, float eps,
                   int K, uint16_t* r_out, uint16_t* __restrict__ X) {
  extern __shared__ __align__(16) uint4 rs[];   // the row's r, K / 8 chunks
  __shared__ float wsum[kNormThreads / 32];
  const int chunks = K / 8;
  const size_t base = (size_t)blockIdx.x * chunks;
  const uint4* hv = reinterpret_cast<const uint4*>(h) + base;
  const uint4* dv = d ? reinterpret_cast<const uint4*>(d) + base : nullptr;
  uint4* rv = r_out ? reinterpret_cast<uint4*>(r_out) + base : nullptr;
  ptx::griddep_launch_dependents();

  float ss = 0.0f;
  for (int c0 = threadIdx.x; c0 < chunks; c0 += kNormThreads * kNormBatch) {
    uint4 a[kNormBatch], b[kNormBatch];
#pragma unroll
    for (int i = 0; i < kNormBatch; ++i) {
      const int c = c0 + i * kNormThreads;
      a[i] = make_uint4(0, 0, 0, 0);
      b[i] = make_uint4(0, 0, 0, 0);
      if (c < chunks) {
        a[i] = hv[c];
        if (dv) b[i] = dv[c];
      }
    }
#pragma unroll
    for (int i = 0; i < kNormBatch; ++i) {
      const int c = c0 + i * kNormThreads;
      if (c < chunks) {
        uint4 r = a[i];
        if (dv) {
          r.x = hadd2_rn(a[i].x, b[i].x);
          r.y = hadd2_rn(a[i].y, b[i].y);
          r.z = hadd2_rn(a[i].z, b[i].z);
          r.w = hadd2_rn(a[i].w, b[i].w);
        }
        rs[c] = r;
        if (rv) rv[c] = r;
        ss = sum_sq2(r.x, ss);
        ss = sum_sq2(r.y, ss);
        ss = sum_sq2(r.z, ss);
        ss = sum_sq2(r.w, ss);
      }
    }
  }

  // Butterfly: every lane ends with the same warp sum; the warps' sums are
  // then added in warp order, so the result does not depend on timing.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) tot += wsum[w];
  const float inv = rms_inv(tot, K, eps);

  const uint4* gv = reinterpret_cast<const uint4*>(gamma);
  uint4* xv = reinterpret_cast<uint4*>(X) + base;
  for (int c = threadIdx.x; c < chunks; c += kNormThreads) {
    const uint4 r = rs[c];
    const uint4 g = __ldg(gv + c);
    uint4 o;
    o.x = scale2(r.x, g.x, inv);
    o.y = scale2(r.y, g.y, inv);
    o.z = scale2(r.z, g.z, inv);
    o.w = scale2(r.w, g.w, inv);
    xv[c] = o;
  }
}

}  // namespace

cudaError_t launch_add_rmsnorm(const uint16_t* h, const uint16_t* d, const uint16_t* gamma, float eps,
                               int N, int K, uint16_t* r_out, uint16_t* X, cudaStream_t stream) {
  const size_t smem = (size_t)K * 2;
  if (smem > 48 * 1024) {
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(add_rmsnorm_kernel), kMaxNormK * 2, smem_set);
    if (e != cudaSuccess) return e;
  }
  add_rmsnorm_kernel<<<(unsigned)N, kNormThreads, smem, stream>>>(h, d, gamma, eps, K, r_out, X);
  return cudaGetLastError();
}

}  // namespace w4a16
