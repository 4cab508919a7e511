// k_classify.cu -- SLA's compressed scores and percentile classification.
//
// SLA page section 3: the pooled Q and K give a compressed attention-weight
// matrix P_c = softmax(pool(Q) pool(K)^T / sqrt(d)); within each query-block row
// the top 5 % positions are labelled critical (1), the bottom 10 % negligible
// (-1), the rest marginal (0).  Softmax is strictly increasing along a row, so
// the labels are taken on the fp64 logits; ties rank the lower key-block index
// first.  Both the logits and the selection are fp64 so that the labels agree
// with an fp64 evaluation of the same definition.
//
// block_logits_kernel: 64x64 output tiles of qbar kbar^T on the fp64 tensor cores.
// classify_rows_kernel: one warp per row; two MSB-first radix selections over
//   order-preserving 64-bit keys (8-bit digits, warp-aggregated histogram
//   counts, stopping once the remaining candidates are exactly the ones
//   needed) find the kc-th largest and kn-th smallest key; one pass in index
//   order applies the
//   thresholds with index tie-breaking and emits the mask row, the ascending
//   critical list, the marginal indicator row (bf16 1/0 for the tensor-core
//   contraction) and, on request, P_c in fp32.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

// dots[bh][i][j] = qbar_i . kbar_j in fp64 on the fp64 tensor cores
// (mma.m8n8k4.f64): one CTA = 4 warps computes a 64x64 tile, each warp a 32x32
// quarter as 4x4 fragments of 8x8.  The ranking of a row does not depend on the
// positive scale 1/sqrt(d), so the kernel stores the plain dot products.
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1]) : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(128)
block_logits_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                    double* __restrict__ dots, int nb, int d) {
  __shared__ double As[64][36];
  __shared__ double Bs[64][36];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const double* A = qbar + (size_t)bh * nb * d;
  const double* B = kbar + (size_t)bh * nb * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wy = warp >> 1, wx = warp & 1;
  double acc[4][4][2];
  #pragma unroll
  for (int a = 0; a < 4; ++a)
    #pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;
  for (int c0 = 0; c0 < d; c0 += 32) {
    for (int e = threadIdx.x; e < 64 * 32; e += 128) {
      const int row = e >> 5, col = e & 31;
      As[row][col] = (i0 + row < nb) ? A[(size_t)(i0 + row) * d + c0 + col] : 0.0;
      Bs[row][col] = (j0 + row < nb) ? B[(size_t)(j0 + row) * d + c0 + col] : 0.0;
    }
    __syncthreads();
    #pragma unroll
    for (int kk = 0; kk < 32; kk += 4) {
      double af[4], bf[4];
      #pragma unroll
      for (int t = 0; t < 4; ++t) {
        af[t] = As[wy * 32 + t * 8 + (lane >> 2)][kk + (lane & 3)];
        bf[t] = Bs[wx * 32 + t * 8 + (lane >> 2)][kk + (lane & 3)];
      }
      #pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        #pragma unroll
        for (int nt = 0; nt < 4; ++nt) dmma_8x8x4(acc[mt][nt], af[mt], bf[nt]);
    }
    __syncthreads();
  }
  #pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int i = i0 + wy * 32 + mt * 8 + (lane >> 2);
    if (i >= nb) continue;
    #pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int j = j0 + wx * 32 + nt * 8 + 2 * (lane & 3);
      double* dst = dots + ((size_t)bh * nb + i) * nb + j;
      if (j < nb) dst[0] = acc[mt][nt][0];
      if (j + 1 < nb) dst[1] = acc[mt][nt][1];
    }
  }
}

// Order-preserving map of an fp64 value onto uint64 (larger value -> larger key);
// -0 is folded onto +0 so that equal values give equal keys.
__device__ __forceinline__ uint64_t order_key(double x) {
  if (x == 0.0) x = 0.0;
  const uint64_t b = (uint64_t)__double_as_longlong(x);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// MSB-first radix selection of the k-th largest (largest=true) or k-th smallest
// key among keys[0..n), 8 bits per pass.  Returns the selection at the level
// `shift` where it was settled: T (the key's bits above `shift`), how many of
// the keys whose bits above `shift` equal T are taken (take), and how many such
// keys there are (eq_total).  The passes stop early once every remaining
// candidate is needed.
__device__ void radix_select(const uint64_t* keys, int n, int k, bool largest, unsigned* hist, int lane,
                             uint64_t& T, int& shift_out, int& take, int& eq_total) {
  uint64_t prefix = 0, pmask = 0;
  int kk = k, last = 0, shift = 56;
  for (;; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint64_t u = j < n ? keys[j] : 0;
      const bool cand = j < n && (u & pmask) == prefix;
      const unsigned bin = (unsigned)((u >> shift) & 255);
      const unsigned act = __ballot_sync(0xFFFFFFFFu, cand);
      if (cand) {
        const unsigned peers = __match_any_sync(act, bin);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], (unsigned)__popc(peers));
      }
    }
    __syncwarp();
    int cnt[8], lsum = 0;
    #pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int bin = largest ? 255 - (lane * 8 + q) : lane * 8 + q;
      cnt[q] = (int)hist[bin];
      lsum += cnt[q];
    }
    const int incl = warp_incl_scan(lsum, lane);
    const int excl = incl - lsum;
    const bool has = excl < kk && incl >= kk;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, has);
    const int src = __ffs(bal) - 1;
    int sel = 0, before = 0;
    if (lane == src) {
      int acc = excl;
      #pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc + cnt[q] >= kk) { sel = largest ? 255 - (lane * 8 + q) : lane * 8 + q; before = acc; break; }
        acc += cnt[q];
      }
    }
    sel = __shfl_sync(0xFFFFFFFFu, sel, src);
    before = __shfl_sync(0xFFFFFFFFu, before, src);
    kk -= before;
    last = (int)hist[sel];
    prefix |= (uint64_t)sel << shift;
    pmask |= (uint64_t)0xFF << shift;
    __syncwarp();
    if (last == kk || shift == 0) break;      // every remaining candidate is needed, or fully resolved
  }
  T = prefix >> shift;
  shift_out = shift;
  take = kk;
  eq_total = last;
}

constexpr int kRowsPerCta = 4;

__global__ void __launch_bounds__(128)
classify_rows_kernel(const double* __restrict__ logits, int rows, int nb, int kc, int kn,
                     int8_t* __restrict__ mask, int32_t* __restrict__ crit_idx, int32_t* __restrict__ crit_cnt,
                     __nv_bfloat16* __restrict__ m01, int ld_m01, float* __restrict__ scores, double sqrt_d) {
  extern __shared__ uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem) + (size_t)warp * nb;
  unsigned* hist = reinterpret_cast<unsigned*>(reinterpret_cast<uint64_t*>(smem) + (size_t)kRowsPerCta * nb) + warp * 256;
  const int row = blockIdx.x * kRowsPerCta + warp;
  if (row >= rows) return;
  const double* lg = logits + (size_t)row * nb;
  double mx = -INFINITY;
  for (int j = lane; j < nb; j += 32) {
    const double x = lg[j];
    keys[j] = order_key(x);
    mx = fmax(mx, x);
  }
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  double sum = 0.0;
  if (scores) {
    for (int j = lane; j < nb; j += 32) sum += exp(lg[j] / sqrt_d - mx / sqrt_d);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  }
  __syncwarp();
  uint64_t Tc = 0, Tn = 0;
  int sc = 0, sn = 0, take_c = 0, eq_c = 0, take_n = 0, eq_n = 0;
  radix_select(keys, nb, kc, true, hist, lane, Tc, sc, take_c, eq_c);
  if (kn > 0) radix_select(keys, nb, kn, false, hist, lane, Tn, sn, take_n, eq_n);
  const unsigned lt_mask = (1u << lane) - 1u;
  int seen_c = 0, seen_n = 0, written = 0;
  for (int base = 0; base < nb; base += 32) {
    const int j = base + lane;
    const bool in = j < nb;
    const uint64_t u = in ? keys[j] : 0;
    const uint64_t uc = u >> sc, un = u >> sn;
    const bool eqc = in && uc == Tc;
    const unsigned bc = __ballot_sync(0xFFFFFFFFu, eqc);
    const bool crit = (in && uc > Tc) || (eqc && seen_c + __popc(bc & lt_mask) < take_c);
    seen_c += __popc(bc);
    bool negl = false;
    if (kn > 0) {
      const bool eqn = in && un == Tn;
      const unsigned bn = __ballot_sync(0xFFFFFFFFu, eqn);
      negl = (in && un < Tn) || (eqn && seen_n + __popc(bn & lt_mask) >= eq_n - take_n);
      seen_n += __popc(bn);
    }
    if (in) {
      const int8_t m = crit ? 1 : (negl ? -1 : 0);
      mask[(size_t)row * nb + j] = m;
      if (m01) m01[(size_t)row * ld_m01 + j] = __float2bfloat16_rn(m == 0 ? 1.f : 0.f);
      if (scores) scores[(size_t)row * nb + j] = (float)(exp(lg[j] / sqrt_d - mx / sqrt_d) / sum);
    }
    const unsigned bcrit = __ballot_sync(0xFFFFFFFFu, crit);
    if (crit) crit_idx[(size_t)row * kc + written + __popc(bcrit & lt_mask)] = j;
    written += __popc(bcrit);
  }
  if (m01)
    for (int j = nb + lane; j < ld_m01; j += 32) m01[(size_t)row * ld_m01 + j] = __float2bfloat16_rn(0.f);
  if (lane == 0) crit_cnt[row] = kc;
}

__global__ void mask_to_m01_kernel(const int8_t* __restrict__ mask, __nv_bfloat16* __restrict__ m01,
                                   int rows, int nb, int ld) {
  const size_t total = (size_t)rows * ld;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t r = e / ld;
    const int j = (int)(e % ld);
    const float v = (j < nb && mask[r * nb + j] == 0) ? 1.f : 0.f;
    m01[e] = __float2bfloat16_rn(v);
  }
}

}  // namespace

cudaError_t launch_block_logits(const double* qbar, const double* kbar, double* logits,
                                int BH, int nb, int d, cudaStream_t st) {
  dim3 grid((nb + 63) / 64, (nb + 63) / 64, BH);
  block_logits_kernel<<<grid, 128, 0, st>>>(qbar, kbar, logits, nb, d);
  return cudaGetLastError();
}

cudaError_t launch_classify_rows(const double* logits, int BH, int nb, int d, int kc, int kn,
                                 int8_t* mask, int32_t* crit_idx, int32_t* crit_cnt,
                                 __nv_bfloat16* m01, int ld_m01, float* scores, cudaStream_t st) {
  const int rows = BH * nb;
  const size_t smem = (size_t)kRowsPerCta * nb * sizeof(uint64_t) + (size_t)kRowsPerCta * 256 * sizeof(unsigned);
  cudaError_t e = cudaFuncSetAttribute(classify_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  classify_rows_kernel<<<(rows + kRowsPerCta - 1) / kRowsPerCta, 128, smem, st>>>(
      logits, rows, nb, kc, kn, mask, crit_idx, crit_cnt, m01, ld_m01, scores, sqrt((double)d));
  return cudaGetLastError();
}

cudaError_t launch_mask_to_m01(const int8_t* mask, __nv_bfloat16* m01, int BH, int nb, int ld_m01,
                               cudaStream_t st) {
  const int rows = BH * nb;
  const size_t total = (size_t)rows * ld_m01;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  mask_to_m01_kernel<<<blocks, 256, 0, st>>>(mask, m01, rows, nb, ld_m01);
  return cudaGetLastError();
}

}  // namespace slr
