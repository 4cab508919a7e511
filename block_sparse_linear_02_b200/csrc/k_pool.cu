// k_pool.cu -- bandwidth-bound pooling kernels.
//
// pool_means_kernel: the per-block mean of Q and of K that feeds SLA's
// compressed score matrix (SLA page, section 3: both Q and K are averaged over
// each token block first).  One CTA reads one 64-token block (16-byte vector
// loads, valid tokens only).  Sums of at most 64 bf16 values are exact in fp64,
// so the mean does not depend on summation order.  It is written as a bf16 pair
// hi + lo (hi = bf16(mean), lo = bf16(mean - hi), 16 significant bits together)
// in the row layout the tensor-core logits GEMM consumes.  With phi_q given, the Q
// pass also writes phi(Q) for every token of the block (elu(Q) + 1, or the softmax
// over the channels of each row; 0 for pad tokens), the operand of the linear branch
// the attention kernel applies.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

__device__ __forceinline__ float phi_elu1_ex2(float x) {
  // elu(x) + 1 = exp(min(x, 0)) + max(x, 0); exp through the exp2 unit (rounded to bf16 after)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fminf(x, 0.f) * 1.4426950408889634f));
  return y + fmaxf(x, 0.f);
}

template <int D>
__global__ void __launch_bounds__(128)
pool_means_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  __nv_bfloat16* __restrict__ qsplit, __nv_bfloat16* __restrict__ ksplit,
                  __nv_bfloat16* __restrict__ phi_q, int phi, SeqShape s) {
  constexpr int kCPR = D / 8;          // 16-byte chunks per row
  constexpr int kRG = 128 / kCPR;      // row groups
  __shared__ double red[kRG][D];
  const int blk = blockIdx.x, bh = blockIdx.y;
  const bool is_q = blockIdx.z == 0;
  const __nv_bfloat16* x = (is_q ? q : k) + ((size_t)bh * s.n_pad + (size_t)blk * kBlock) * D;
  __nv_bfloat16* out = (is_q ? qsplit : ksplit) + ((size_t)bh * s.n_blocks + blk) * 3 * D;
  const int chunk = threadIdx.x % kCPR, rg = threadIdx.x / kCPR;
  const int nvalid = block_valid_count(s, blk);   // valid tokens form a prefix of the block
  // all of a thread's rows are loaded before any is summed (64 / kRG 16-byte loads in flight)
  constexpr int kRows = kBlock / kRG;
  uint4 u[kRows];
  #pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int r = rg + k * kRG;
    u[k] = r < nvalid ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)r * D + chunk * 8)) : make_uint4(0, 0, 0, 0);
  }
  if (is_q && phi_q) {
    uint4* dst = reinterpret_cast<uint4*>(phi_q + ((size_t)bh * s.n_pad + (size_t)blk * kBlock) * D);
    #pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int r = rg + k * kRG;
      const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
      float f[8];
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
      }
      if (phi == SLR_PHI_SOFTMAX) {
        row_softmax8<kCPR>(f);                   // the kCPR lanes of row r (uniform: phi is per launch)
      } else {
        #pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = phi_elu1_ex2(f[i]);
      }
      uint32_t o[4];
      #pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = r < nvalid ? pack_bf16(f[2 * i], f[2 * i + 1]) : 0u;
      dst[(size_t)r * (D / 8) + chunk] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  double acc[8];
  #pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  #pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += (double)bf16_lo(w[i]);
      acc[2 * i + 1] += (double)bf16_hi(w[i]);
    }
  }
  #pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][chunk * 8 + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 128) {
    double sum = 0.0;
    #pragma unroll
    for (int g = 0; g < kRG; ++g) sum += red[g][c];
    const double mean = sum / (double)nvalid;
    const __nv_bfloat16 hi = __double2bfloat16(mean);
    const __nv_bfloat16 lo = __double2bfloat16(mean - (double)__bfloat162float(hi));
    // Q rows [hi | hi | lo], K rows [hi | lo | hi]: their dot product is
    // qh.kh + qh.kl + ql.kh, the pooled logit up to the tiny ql.kl term
    out[c] = hi;
    out[D + c] = is_q ? hi : lo;
    out[2 * D + c] = is_q ? lo : hi;
  }
}

}  // namespace

cudaError_t launch_pool_means(const void* q, const void* k, void* qsplit, void* ksplit, void* phi_q, int phi,
                              int BH, int d, SeqShape s, cudaStream_t st) {
  dim3 grid(s.n_blocks, BH, 2);
  auto* qs = static_cast<__nv_bfloat16*>(qsplit);
  auto* ks = static_cast<__nv_bfloat16*>(ksplit);
  auto* pq = static_cast<__nv_bfloat16*>(phi_q);
  if (d == 128)
    pool_means_kernel<128><<<grid, 128, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qs, ks, pq, phi, s);
  else
    pool_means_kernel<64><<<grid, 128, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qs, ks, pq, phi, s);
  return cudaGetLastError();
}

}  // namespace slr
