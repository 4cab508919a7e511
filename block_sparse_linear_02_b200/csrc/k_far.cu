// k_far.cu -- the passes over K and V (and Q) that precede the tile attention kernels.
//
// The tile kernels load each 4x4x4 key tile as 64 consecutive rows, so K and V are first
// written in tile-major order: tile (th * TW + tw) * TF + tf takes rows [64 tile,
// 64 tile + 64), its tokens in (f, h, w) raster order inside the tile.
//
//   tile_major_kernel   K and V copied into tile-major order (sliding tile mask).
//   rope_table_kernel   cos / sin of the 3-D rotary embedding for every (axis coordinate,
//                       channel pair): RoPeSLR page, the neighbourhood branch encodes
//                       relative position with RoPE.
//   far_rows_kernel     RoPeSLR mode, one CTA per raster row (f, h) of one head and one of
//                       K, V, Q: K and V are written tile-major (K rotated first with RoPE),
//                       Q rotated in raster order (RoPE only), and the row's K and V values
//                       are summed per far-field cell segment (aixinbiao page: K and V
//                       compressed by token mean-pooling into a small set).
//   far_finish_kernel   the cell means from those row sums, rounded to bf16 because they
//                       are tensor-core operands of the attention kernel.
//
// Every CTA of the row passes handles one short raster row, so the grid holds thousands of
// CTAs, each thread with four 16-byte loads in flight.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

// Row of raster token (f, h, w) in tile-major order.
__device__ __forceinline__ int tile_major_row(int f, int h, int w, int TF, int TW) {
  return ((((h >> 2) * TW + (w >> 2)) * TF + (f >> 2)) << 6) + ((f & 3) << 4) + ((h & 3) << 2) + (w & 3);
}

// One CTA per (raster row (f, h), head, tensor).
template <int D>
__global__ void __launch_bounds__(256)
tile_major_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                  __nv_bfloat16* __restrict__ kt, __nv_bfloat16* __restrict__ vt, int F, int Hh, int Ww) {
  constexpr int kCPR = D / 8;              // 16-byte chunks per token
  const int row = blockIdx.x, bh = blockIdx.y;
  const int f = row / Hh, h = row % Hh;
  const size_t n = (size_t)F * Hh * Ww;
  const __nv_bfloat16* x = (blockIdx.z == 0 ? k : v) + ((size_t)bh * n + (size_t)row * Ww) * D;
  __nv_bfloat16* y = (blockIdx.z == 0 ? kt : vt) + (size_t)bh * n * D;
  const int TF = F >> 2, TW = Ww >> 2;
  for (int i = threadIdx.x; i < Ww * kCPR; i += blockDim.x) {
    const int w = i / kCPR, c = i % kCPR;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + (size_t)w * D + c * 8));
    *reinterpret_cast<uint4*>(y + (size_t)tile_major_row(f, h, w, TF, TW) * D + c * 8) = u;
  }
}

// Channel pairs of the 3-D rotary embedding: with P = D/2 pairs the frame axis takes the
// first P - 2 floor(P/3), the height and width axes floor(P/3) each.
template <int D>
struct RopeSplit {
  static constexpr int kPairs = D / 2, kH = kPairs / 3, kW = kPairs / 3, kF = kPairs - kH - kW;
};

// (cos, sin) of pos * 10000^(-i/n) for pair i of an axis group of n pairs: the frame table
// [F][kF], then the height table [Hh][kH], then the width table [Ww][kW].
template <int D>
__global__ void rope_table_kernel(float2* __restrict__ tab, int F, int Hh, int Ww) {
  using R = RopeSplit<D>;
  const int nf = F * R::kF, nh = Hh * R::kH, n_tab = nf + nh + Ww * R::kW;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_tab; e += gridDim.x * blockDim.x) {
    int pos, i, np;
    if (e < nf) { pos = e / R::kF; i = e % R::kF; np = R::kF; }
    else if (e < nf + nh) { pos = (e - nf) / R::kH; i = (e - nf) % R::kH; np = R::kH; }
    else { pos = (e - nf - nh) / R::kW; i = (e - nf - nh) % R::kW; np = R::kW; }
    // 10000^(-i/n) = 2^(-(i/n) log2 10000)
    const float ang = (float)pos * exp2f(-(float)i / (float)np * 13.287712379549449f);
    float sn, cs;
    sincosf(ang, &sn, &cs);
    tab[e] = make_float2(cs, sn);
  }
}

// z = 0: K, 1: V, 2: Q (with RoPE only).  The CTA's Ww tokens pass through shared memory as
// the bf16 values written out, and the K / V ones are summed per cell segment of cw tokens
// in a fixed order into part[z][bh][row][Ww / cw][D] (fp32).
template <int D>
__global__ void __launch_bounds__(256)
far_rows_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ qr,
                __nv_bfloat16* __restrict__ kt, __nv_bfloat16* __restrict__ vt,
                const float2* __restrict__ tab, float* __restrict__ part, int F, int Hh, int Ww, int cw,
                int rope) {
  using R = RopeSplit<D>;
  constexpr int kCPR = D / 8;              // 16-byte chunks per token = 4 channel pairs each
  extern __shared__ __nv_bfloat16 row_vals[];   // [Ww][D]
  const int row = blockIdx.x, bh = blockIdx.y, z = blockIdx.z;
  const int f = row / Hh, h = row % Hh;
  const size_t n = (size_t)F * Hh * Ww;
  const __nv_bfloat16* x = (z == 0 ? k : z == 1 ? v : q) + ((size_t)bh * n + (size_t)row * Ww) * D;
  __nv_bfloat16* y = (z == 0 ? kt : z == 1 ? vt : qr) + (size_t)bh * n * D;
  const bool rotate = rope && z != 1;      // uniform over the CTA
  const bool pool = z != 2;
  const int TF = F >> 2, TW = Ww >> 2;
  // a thread keeps one 16-byte chunk c of every token it handles (blockDim is a multiple of
  // kCPR): the frame and height angles of its pairs are fixed for the CTA, the width ones
  // depend on the token
  constexpr int kTokStep = 256 / kCPR;     // tokens per pass of the CTA
  const int c = threadIdx.x % kCPR;
  float2 cs_fixed[4];
  int w_pair[4];                           // width pair index, or -1 for a frame / height pair
  #pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int pr = c * 4 + e;
    cs_fixed[e] = make_float2(1.f, 0.f);
    w_pair[e] = -1;
    if (rotate) {
      if (pr < R::kF) cs_fixed[e] = __ldg(tab + f * R::kF + pr);
      else if (pr < R::kF + R::kH) cs_fixed[e] = __ldg(tab + F * R::kF + h * R::kH + (pr - R::kF));
      else w_pair[e] = pr - R::kF - R::kH;
    }
  }
  const float2* tab_w = tab + F * R::kF + Hh * R::kH;
  // four tokens' loads in flight per thread
  for (int w_base = threadIdx.x / kCPR; w_base < Ww; w_base += 4 * kTokStep) {
    uint4 u[4];
    #pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int w = w_base + m * kTokStep;
      u[m] = w < Ww ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)w * D + c * 8)) : make_uint4(0, 0, 0, 0);
    }
    #pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int w = w_base + m * kTokStep;
      if (w >= Ww) break;
      uint32_t wd[4] = {u[m].x, u[m].y, u[m].z, u[m].w};
      if (rotate) {
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 cs = w_pair[e] < 0 ? cs_fixed[e] : __ldg(tab_w + w * R::kW + w_pair[e]);
          const float a = bf16_lo(wd[e]), b = bf16_hi(wd[e]);
          wd[e] = pack_bf16(a * cs.x - b * cs.y, a * cs.y + b * cs.x);
        }
      }
      const uint4 o = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      const size_t dst = z == 2 ? (size_t)row * Ww + w : (size_t)tile_major_row(f, h, w, TF, TW);
      *reinterpret_cast<uint4*>(y + dst * D + c * 8) = o;
      if (pool) *reinterpret_cast<uint4*>(row_vals + w * D + c * 8) = o;
    }
  }
  if (!pool) return;
  __syncthreads();
  const int segs = Ww / cw;
  float* out = part + (((size_t)z * gridDim.y + bh) * gridDim.x + row) * segs * D;
  for (int i = threadIdx.x; i < segs * D; i += blockDim.x) {
    const int s = i / D, ch = i % D;
    float sum = 0.f;
    for (int w = s * cw; w < (s + 1) * cw; ++w) sum += __bfloat162float(row_vals[w * D + ch]);
    out[i] = sum;
  }
}

// One CTA of D threads per (cell, head, tensor): the mean over the cell's cf x ch row sums.
template <int D>
__global__ void __launch_bounds__(D)
far_finish_kernel(const float* __restrict__ part, __nv_bfloat16* __restrict__ kf, __nv_bfloat16* __restrict__ vf,
                  int F, int Hh, int Ww, int cf, int ch, int cw) {
  const int cell = blockIdx.x, bh = blockIdx.y, z = blockIdx.z, BH = gridDim.y;
  const int gh = Hh / ch, gw = Ww / cw, segs = Ww / cw;
  const int c_f = cell / (gh * gw), c_h = (cell / gw) % gh, c_w = cell % gw;
  const float* base = part + ((size_t)z * BH + bh) * (size_t)F * Hh * segs * D;
  float sum = 0.f;
  for (int df = 0; df < cf; ++df)
    for (int dh = 0; dh < ch; ++dh) {
      const int row = (c_f * cf + df) * Hh + c_h * ch + dh;
      sum += base[((size_t)row * segs + c_w) * D + threadIdx.x];
    }
  __nv_bfloat16* out = (z == 0 ? kf : vf) + ((size_t)bh * gridDim.x + cell) * D;
  out[threadIdx.x] = __float2bfloat16_rn(sum / (float)(cf * ch * cw));
}

template <int D>
cudaError_t far_field_d(const void* q, const void* k, const void* v, void* qr, void* kt, void* vt, void* kf,
                        void* vf, float2* tab, float* part, int BH, int F, int Hh, int Ww, int cf, int ch, int cw,
                        int rope, cudaStream_t st) {
  using bf = __nv_bfloat16;
  if (rope) {
    using R = RopeSplit<D>;
    const int n_tab = F * R::kF + Hh * R::kH + Ww * R::kW;
    rope_table_kernel<D><<<(n_tab + 255) / 256, 256, 0, st>>>(tab, F, Hh, Ww);
  }
  const size_t smem = (size_t)Ww * D * sizeof(bf);
  static unsigned long long attr_set = 0;          // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && (dev >= 64 || !(attr_set & (1ull << dev)))) {
    const cudaError_t e = cudaFuncSetAttribute(far_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)kFarRowBytesMax);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  dim3 grid(F * Hh, BH, rope ? 3 : 2);
  far_rows_kernel<D><<<grid, 256, smem, st>>>(static_cast<const bf*>(q), static_cast<const bf*>(k),
                                              static_cast<const bf*>(v), static_cast<bf*>(qr), static_cast<bf*>(kt),
                                              static_cast<bf*>(vt), tab, part, F, Hh, Ww, cw, rope);
  const int ncells = (F / cf) * (Hh / ch) * (Ww / cw);
  far_finish_kernel<D><<<dim3(ncells, BH, 2), D, 0, st>>>(part, static_cast<bf*>(kf), static_cast<bf*>(vf), F, Hh,
                                                           Ww, cf, ch, cw);
  return cudaGetLastError();
}

}  // namespace

size_t far_rope_table_bytes(int d, int F, int Hh, int Ww) {
  const int pairs = d / 2, hw = pairs / 3;
  return ((size_t)F * (pairs - 2 * hw) + ((size_t)Hh + Ww) * hw) * sizeof(float2);
}

size_t far_partial_bytes(int BH, int d, int F, int Hh, int Ww, int cw) {
  return 2 * (size_t)BH * F * Hh * (Ww / cw) * d * sizeof(float);
}

cudaError_t launch_tile_major(const void* k, const void* v, void* kt, void* vt, int BH, int d, int F, int Hh,
                              int Ww, cudaStream_t st) {
  dim3 grid(F * Hh, BH, 2);
  auto* k_ = static_cast<const __nv_bfloat16*>(k);
  auto* v_ = static_cast<const __nv_bfloat16*>(v);
  auto* kt_ = static_cast<__nv_bfloat16*>(kt);
  auto* vt_ = static_cast<__nv_bfloat16*>(vt);
  if (d == 128) tile_major_kernel<128><<<grid, 256, 0, st>>>(k_, v_, kt_, vt_, F, Hh, Ww);
  else tile_major_kernel<64><<<grid, 256, 0, st>>>(k_, v_, kt_, vt_, F, Hh, Ww);
  return cudaGetLastError();
}

cudaError_t launch_far_field(const void* q, const void* k, const void* v, void* qr, void* kt, void* vt, void* kf,
                             void* vf, void* tab, void* part, int BH, int d, int F, int Hh, int Ww, int cf, int ch,
                             int cw, int rope, cudaStream_t st) {
  if ((size_t)Ww * d * sizeof(__nv_bfloat16) > kFarRowBytesMax) return cudaErrorInvalidValue;
  auto* t = static_cast<float2*>(tab);
  auto* pp = static_cast<float*>(part);
  return d == 128 ? far_field_d<128>(q, k, v, qr, kt, vt, kf, vf, t, pp, BH, F, Hh, Ww, cf, ch, cw, rope, st)
                  : far_field_d<64>(q, k, v, qr, kt, vt, kf, vf, t, pp, BH, F, Hh, Ww, cf, ch, cw, rope, st);
}

}  // namespace slr
