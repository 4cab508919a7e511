// k_pool.cu -- bandwidth-bound pooling kernels.
//
// pool_means_kernel: the per-block mean of Q and of K that feeds SLA's
// compressed score matrix (SLA page, section 3: both Q and K are averaged over
// each token block first).  One CTA reads one 64-token block (16-byte vector
// loads, valid tokens only).  Sums of at most 64 bf16 values are exact in fp64,
// so the mean does not depend on summation order.  It is written as a bf16 pair
// hi + lo (hi = bf16(mean), lo = bf16(mean - hi), 16 significant bits together)
// in the row layout the tensor-core logits GEMM consumes.  With phi_q given, the Q
// pass also writes phi(Q) = elu(Q) + 1 for every token of the block (0 for pad
// tokens), the operand of the linear branch the attention kernel applies.
//
// far_pool_kernel: the far field of the RoPeSLR gated mode -- K and V averaged
// over cells of (cf, ch, cw) raster tokens (aixinbiao page: K and V compressed
// by token mean-pooling into a small low-rank set), rounded to bf16 because
// they are tensor-core operands of the attention kernel; with the 3-D rotary
// embedding the same pass rotates Q and K, so each is read from HBM once.  The same pass
// writes K (rotated) and V in the tile-major order the tile attention kernel loads.
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

// Row of raster token (f, h, w) in the tile-major order of 4x4x4 tiles: tile
// (th * TW + tw) * TF + tf, and inside it (f % 4, h % 4, w % 4) in raster order.
__device__ __forceinline__ int tile_major_row(int f, int h, int w, int TF, int TW) {
  return ((((h >> 2) * TW + (w >> 2)) * TF + (f >> 2)) << 6) + ((f & 3) << 4) + ((h & 3) << 2) + (w & 3);
}

// K and V of a raster (F, Hh, Ww) sequence copied into tile-major order, so that the
// attention kernel loads each 4x4x4 key tile as 64 consecutive rows (one 16 KB box per
// 64 channels) instead of gathering 16 runs of 4 tokens.  One CTA per (raster row (f, h),
// head, tensor); the row's Ww tokens are 4-token runs of Ww / 4 tiles.
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

// One CTA per (cell, head, tensor): z = 0 K, 1 V, 2 Q (the last only with the rotary
// embedding).  V is averaged over the cell; with the embedding, K is rotated, written out
// and averaged as rotated (the far field pools the rotated keys), and Q is rotated and
// written out.  Pair i of an axis group of n pairs turns by pos * 10000^(-i/n), pos the
// token's coordinate on that axis (RoPeSLR page: RoPE encodes the relative position in
// the neighbourhood); the cos / sin of every (coordinate inside the cell, pair) are
// tabulated once per CTA in shared memory.
template <int D>
__global__ void __launch_bounds__(128)
far_pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ qr,
                __nv_bfloat16* __restrict__ kt, __nv_bfloat16* __restrict__ vt, __nv_bfloat16* __restrict__ kf,
                __nv_bfloat16* __restrict__ vf, int F, int Hh, int Ww, int cf, int ch, int cw, int rope) {
  using R = RopeSplit<D>;
  constexpr int kCPR = D / 8;              // 16-byte chunks per row = 4 channel pairs each
  constexpr int kRG = 128 / kCPR;
  __shared__ float red[kRG][D];
  extern __shared__ float2 cs_tab[];       // [cf][kF], then [ch][kH], then [cw][kW]: (cos, sin)
  const int cell = blockIdx.x, bh = blockIdx.y, z = blockIdx.z;
  const int gh = Hh / ch, gw = Ww / cw;
  const int c_f = cell / (gh * gw), c_h = (cell / gw) % gh, c_w = cell % gw;
  const size_t n = (size_t)F * Hh * Ww;
  const __nv_bfloat16* x = (z == 0 ? k : z == 1 ? v : q) + (size_t)bh * n * D;
  const bool rotate = rope && z != 1;
  const bool pool = z != 2;
  // K and V (rotated K) leave in tile-major order, rotated Q in raster order
  __nv_bfloat16* xo = (z == 0 ? kt : z == 1 ? vt : qr) + (size_t)bh * n * D;
  const int TF = F >> 2, TW = Ww >> 2;
  const int chunk = threadIdx.x % kCPR, rg = threadIdx.x / kCPR;
  const int per_cell = cf * ch * cw;
  int tab_off[4] = {0, 0, 0, 0}, tab_stride[4] = {0, 0, 0, 0}, axis[4] = {0, 0, 0, 0};
  if (rotate) {                            // uniform over the CTA
    const int nf = cf * R::kF, nh = ch * R::kH, n_tab = nf + nh + cw * R::kW;
    for (int e = threadIdx.x; e < n_tab; e += blockDim.x) {
      int pos, i, np;
      if (e < nf) { pos = c_f * cf + e / R::kF; i = e % R::kF; np = R::kF; }
      else if (e < nf + nh) { pos = c_h * ch + (e - nf) / R::kH; i = (e - nf) % R::kH; np = R::kH; }
      else { pos = c_w * cw + (e - nf - nh) / R::kW; i = (e - nf - nh) % R::kW; np = R::kW; }
      // 10000^(-i/n) = 2^(-(i/n) log2 10000)
      const float ang = (float)pos * exp2f(-(float)i / (float)np * 13.287712379549449f);
      float sn, cs;
      sincosf(ang, &sn, &cs);
      cs_tab[e] = make_float2(cs, sn);
    }
    #pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int pr = chunk * 4 + e;
      if (pr < R::kF) { axis[e] = 0; tab_off[e] = pr; tab_stride[e] = R::kF; }
      else if (pr < R::kF + R::kH) { axis[e] = 1; tab_off[e] = nf + pr - R::kF; tab_stride[e] = R::kH; }
      else { axis[e] = 2; tab_off[e] = nf + nh + pr - R::kF - R::kH; tab_stride[e] = R::kW; }
    }
    __syncthreads();
  }
  float acc[8];
  #pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  // rows rg, rg + kRG, ... of the cell, four loads in flight per batch; the (frame, row,
  // column) offsets inside the cell advance incrementally
  int df = rg / (ch * cw), dh = (rg / cw) % ch, dw = rg % cw;
  constexpr int kBatch = 4;
  for (int r0 = rg; r0 < per_cell; r0 += kBatch * kRG) {
    uint4 u[kBatch];
    int pos[kBatch][3];
    size_t off[kBatch], dst[kBatch];
    #pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      pos[b][0] = df; pos[b][1] = dh; pos[b][2] = dw;
      const int f = c_f * cf + df, h = c_h * ch + dh, w = c_w * cw + dw;
      off[b] = (((size_t)f * Hh + h) * Ww + w) * D + chunk * 8;
      dst[b] = z == 2 ? off[b] : (size_t)tile_major_row(f, h, w, TF, TW) * D + chunk * 8;
      u[b] = r0 + b * kRG < per_cell ? __ldg(reinterpret_cast<const uint4*>(x + off[b])) : make_uint4(0, 0, 0, 0);
      dw += kRG;
      while (dw >= cw) {
        dw -= cw;
        if (++dh == ch) { dh = 0; ++df; }
      }
    }
    #pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      uint32_t w[4] = {u[b].x, u[b].y, u[b].z, u[b].w};
      if (r0 + b * kRG < per_cell) {
        if (rotate) {
          #pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int pe = axis[e] == 0 ? pos[b][0] : axis[e] == 1 ? pos[b][1] : pos[b][2];
            const float2 c = cs_tab[tab_off[e] + pe * tab_stride[e]];
            const float a = bf16_lo(w[e]), bb = bf16_hi(w[e]);
            w[e] = pack_bf16(a * c.x - bb * c.y, a * c.y + bb * c.x);
          }
        }
        *reinterpret_cast<uint4*>(xo + dst[b]) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (pool) {                          // rows past the cell loaded as zeros
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += bf16_lo(w[i]);
          acc[2 * i + 1] += bf16_hi(w[i]);
        }
      }
    }
  }
  if (!pool) return;                       // uniform over the CTA
  __nv_bfloat16* out = (z == 0 ? kf : vf) + ((size_t)bh * gridDim.x + cell) * D;
  #pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][chunk * 8 + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 128) {
    float sum = 0.f;
    #pragma unroll
    for (int g = 0; g < kRG; ++g) sum += red[g][c];
    out[c] = __float2bfloat16_rn(sum / (float)per_cell);
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

size_t far_pool_table_bytes(int d, int cf, int ch, int cw) {
  const int pairs = d / 2, hw = pairs / 3;
  return (size_t)((size_t)cf * (pairs - 2 * hw) + ((size_t)ch + cw) * hw) * sizeof(float2);
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

cudaError_t launch_far_pool(const void* q, const void* k, const void* v, void* qr, void* kt, void* vt, void* kf,
                            void* vf, int BH, int d, int F, int Hh, int Ww, int cf, int ch, int cw, int rope,
                            cudaStream_t st) {
  const int ncells = (F / cf) * (Hh / ch) * (Ww / cw);
  dim3 grid(ncells, BH, rope ? 3 : 2);
  const size_t tab = rope ? far_pool_table_bytes(d, cf, ch, cw) : 0;
  if (tab > kFarPoolTableMax) return cudaErrorInvalidValue;
  auto* q_ = static_cast<const __nv_bfloat16*>(q);
  auto* k_ = static_cast<const __nv_bfloat16*>(k);
  auto* v_ = static_cast<const __nv_bfloat16*>(v);
  auto* qr_ = static_cast<__nv_bfloat16*>(qr);
  auto* kt_ = static_cast<__nv_bfloat16*>(kt);
  auto* vt_ = static_cast<__nv_bfloat16*>(vt);
  auto* kf_ = static_cast<__nv_bfloat16*>(kf);
  auto* vf_ = static_cast<__nv_bfloat16*>(vf);
  if (d == 128)
    far_pool_kernel<128><<<grid, 128, tab, st>>>(q_, k_, v_, qr_, kt_, vt_, kf_, vf_, F, Hh, Ww, cf, ch, cw, rope);
  else
    far_pool_kernel<64><<<grid, 128, tab, st>>>(q_, k_, v_, qr_, kt_, vt_, kf_, vf_, F, Hh, Ww, cf, ch, cw, rope);
  return cudaGetLastError();
}

}  // namespace slr
