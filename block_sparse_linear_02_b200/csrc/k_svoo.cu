// k_svoo.cu -- SVOO's online bidirectional co-clustering and the reordering around
// the attention over the co-clustered blocks.
//
// SVOO summary (gist.science, arXiv 2603.18636), section 3, stage 2: query and key
// centres start from sampled anchor tokens; step A gives every key an affinity vector
// (its dot products with the query centres) and moves it to the key centre whose
// affinity vector is nearest; step B does the same for the queries against the
// updated key centres; a few iterations give aligned blocks of queries and keys.
//
// With R the centres of the other side (rows R_m) and s_n an own centre, the squared
// distance between the affinity vectors of token x and of s_n is
//     |R x - R s_n|^2 = |R x|^2 - 2 x . u_n + b_n,   u_n = R^T R s_n,  b_n = |R s_n|^2,
// and |R x|^2 is the same for every n.  So one step is:
//   svoo_metric_kernel   u_n and b_n per own centre, in fp64 (tiny: C x C x d);
//                        u_n is stored as three bf16 terms hi + mid + lo (24 bits)
//   svoo_assign_kernel   the scores b_n - 2 x . u_n of 128 tokens against every centre
//                        as one tcgen05 GEMM (M = 128 tokens, N = centres, K = 3d over
//                        the three terms, fp32 accumulation in TMEM), then the argmin of
//                        each row (ties to the lower centre) and the label histogram of
//                        each 1024-token chunk (one CTA per chunk: a ring of token tiles,
//                        scores double-buffered in TMEM)
//   svoo_scan_kernel     bucket offsets of every 1024-token chunk (exclusive scan)
//   svoo_scatter_kernel  the stable order: position -> token, by ascending label and
//                        then token index (the counting sort's second pass)
//   svoo_piece_kernel    fp64 sums of pieces of 256 consecutive positions of one cluster
//   svoo_finalize_kernel each centre becomes the mean of its tokens (its pieces added in
//                        order); an empty cluster keeps its centre
// Every kernel is deterministic (no floating-point atomics), so a call repeated on the
// same inputs returns the same labels.  Pad tokens take the label C and end the order.
//
// svoo_gather_kernel / svoo_scatter_rows_kernel: the rows of q, k, v in the co-clustered
// order, and the output rows back to the token order.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

constexpr int kAsgRows = 128;         // tokens per assignment tile (the MMA's M)
constexpr int kSortChunk = 1024;      // tokens per histogram / scatter chunk
constexpr int kScatterThreads = 256;

// ------------------------------------------------------------------ anchors
// centres[bh][n] = x[bh][anchor[bh][n]] for n < C, 0 for C <= n < Cp.
__global__ void svoo_anchor_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ anchor,
                                   float* __restrict__ centres, int C, int Cp, int d, SeqShape s, int* status) {
  const int n = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  float v = 0.f;
  if (n < C) {
    const int t = anchor[(size_t)bh * C + n];
    if (t >= 0 && t < s.n_pad && token_valid(s, t)) {
      v = __bfloat162float(x[((size_t)bh * s.n_pad + t) * d + c]);
    } else if (c == 0) {
      atomicCAS(status, 0, kErrIndex);
    }
  }
  centres[((size_t)bh * Cp + n) * d + c] = v;
}

// ------------------------------------------------------------------ metric
// For own centre n (< Cs): a_m = R_m . s_n over the Cr centres of the other side,
// u_n = sum_m a_m R_m, b_n = sum_m a_m^2, all in fp64 with a fixed summation order.
// The Cr x d rows of R are staged in shared memory first (one coalesced pass).
// u_n is written as bf16 hi | mid | lo rows of 3d columns; rows n >= Cs are zero.
__global__ void __launch_bounds__(128) svoo_metric_kernel(const float* __restrict__ R, int Cr, int Cpr,
                                                          const float* __restrict__ S, int Cs, int Cps, int d,
                                                          __nv_bfloat16* __restrict__ ub, float* __restrict__ bias) {
  extern __shared__ float4 sR4[];           // Cr x d fp32
  __shared__ double s_n[128];
  __shared__ double a[128];
  const float* sR = reinterpret_cast<const float*>(sR4);
  const int n = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __nv_bfloat16* row = ub + ((size_t)bh * Cps + n) * 3 * d;
  if (n >= Cs) {
    for (int c = tid; c < 3 * d; c += blockDim.x) row[c] = __float2bfloat16_rn(0.f);
    if (tid == 0) bias[(size_t)bh * Cps + n] = 0.f;
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(R + (size_t)bh * Cpr * d);
  for (int i = tid; i < Cr * d / 4; i += blockDim.x) sR4[i] = src[i];
  if (tid < d) s_n[tid] = (double)S[((size_t)bh * Cps + n) * d + tid];
  __syncthreads();
  for (int m = warp; m < Cr; m += 4) {
    double p = 0.0;
    for (int c = lane; c < d; c += 32) p += (double)sR[m * d + c] * s_n[c];
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xFFFFFFFFu, p, off);
    if (lane == 0) a[m] = p;
  }
  __syncthreads();
  if (tid < d) {
    double u = 0.0;
    for (int m = 0; m < Cr; ++m) u += a[m] * (double)sR[m * d + tid];
    const __nv_bfloat16 hi = __double2bfloat16(u);
    const double r1 = u - (double)__bfloat162float(hi);
    const __nv_bfloat16 mid = __double2bfloat16(r1);
    const __nv_bfloat16 lo = __double2bfloat16(r1 - (double)__bfloat162float(mid));
    row[tid] = hi;
    row[d + tid] = mid;
    row[2 * d + tid] = lo;
  }
  if (tid == 0) {
    double b = 0.0;
    for (int m = 0; m < Cr; ++m) b += a[m] * a[m];
    bias[(size_t)bh * Cps + n] = (float)b;
  }
}

// ------------------------------------------------------------------ assignment
// One CTA per 1024-token chunk of one head (8 tiles of 128 tokens), one CTA per SM.
// Shared memory (offsets from a 1024-byte aligned base):
//   X  a ring of nst token tiles (4, or 3 when the metric takes 128 rows), each D/64
//      chunks of 128 rows x 64 bf16 (16 KB),
//      128-byte swizzled
//   U  3D/64 chunks of Cp centre rows x 64 bf16: the hi chunks, the mid chunks, the lo
//      chunks (loaded once: the chunk's head has one metric)
//   then the Cp biases, the label histogram, the mbarriers, the TMEM slot, the abort flag
// Thread 0 loads and issues the MMAs; tile i's scores go to TMEM columns (i & 1) * Cp, so
// that the four warps' argmin of tile i - 1 overlaps the MMAs of tile i, and the load of
// tile i + nst - 1 is issued as soon as the MMAs of tile i - 1 have read their stage.
constexpr int kMaxClusters = 128;
constexpr int kHistSlots = 160;       // >= kMaxClusters + 1 buckets
constexpr int kAsgTiles = kSortChunk / kAsgRows;
constexpr int kXStagesMax = 4;
constexpr size_t kAsgSmemCap = 200 * 1024;   // a fourth stage only below this
template <int D>
struct AsgLayout {
  static constexpr int kAChunks = D / 64;
  static constexpr int kBChunks = 3 * D / 64;
  static constexpr int kAChunkBytes = kAsgRows * 128;
  static constexpr int kXBytes = kAChunks * kAChunkBytes;
  __host__ __device__ static size_t b_chunk_bytes(int Cp) { return (size_t)Cp * 128; }
  __host__ __device__ static size_t u_off(int nst) { return (size_t)nst * kXBytes; }
  __host__ __device__ static size_t bias_off(int Cp, int nst) { return u_off(nst) + kBChunks * b_chunk_bytes(Cp); }
  __host__ __device__ static size_t bytes(int Cp, int nst) {
    return bias_off(Cp, nst) + kMaxClusters * 4 + kHistSlots * 4 + 128 + 1024;
  }
  static int stages(int Cp) { return bytes(Cp, kXStagesMax) <= kAsgSmemCap ? kXStagesMax : kXStagesMax - 1; }
};

template <int D>
__global__ void __launch_bounds__(128, 1) svoo_assign_kernel(const __grid_constant__ CUtensorMap tmX,
                                                             const __grid_constant__ CUtensorMap tmU,
                                                             const float* __restrict__ bias, int C, int Cp,
                                                             int32_t* __restrict__ labels,
                                                             int32_t* __restrict__ counts, int n_chunks, SeqShape s,
                                                             int nst, int* status) {
  using L = AsgLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t b_chunk = (uint32_t)L::b_chunk_bytes(Cp);
  uint8_t* sX = smem;
  uint8_t* sU = smem + L::u_off(nst);
  float* sbias = reinterpret_cast<float*>(smem + L::bias_off(Cp, nst));
  int* hist = reinterpret_cast<int*>(sbias + kMaxClusters);
  uint64_t* x_full = reinterpret_cast<uint64_t*>(hist + kHistSlots);   // [kXStagesMax]
  uint64_t* u_full = x_full + kXStagesMax;
  uint64_t* mma_done = u_full + 1;                                     // [2]
  uint64_t* drain = mma_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_base = chunk * kSortChunk;
  int tiles = (s.n_pad - m_base + kAsgRows - 1) / kAsgRows;
  if (tiles > kAsgTiles) tiles = kAsgTiles;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStagesMax; ++i) mbar_init(&x_full[i], 1);
    mbar_init(u_full, 1);
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < Cp; i += blockDim.x) sbias[i] = bias[(size_t)bh * Cp + i];
  for (int i = threadIdx.x; i <= C; i += blockDim.x) hist[i] = 0;
  if (warp == 0) { tmem_alloc(tmem_slot, (uint32_t)(2 * Cp)); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t id = idesc_bf16(kAsgRows, Cp, false, false);
  int issued = 0, landed = 0;              // thread 0: token tiles loaded / waited for
  auto load_x = [&](int i) {
    uint64_t* bar = &x_full[i % nst];
    mbar_arrive_expect_tx(bar, (uint32_t)L::kXBytes);
    #pragma unroll
    for (int c = 0; c < L::kAChunks; ++c)
      tma_load_3d(sX + (i % nst) * L::kXBytes + c * L::kAChunkBytes, &tmX, bar, c * 64, m_base + i * kAsgRows, bh);
    ++issued;
  };
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(u_full, (uint32_t)(L::kBChunks * b_chunk));
    #pragma unroll
    for (int c = 0; c < L::kBChunks; ++c) tma_load_3d(sU + c * b_chunk, &tmU, u_full, c * 64, 0, bh);
    for (int i = 0; i < nst - 1 && i < tiles; ++i) load_x(i);
  }

  // labels of tile j from TMEM buffer j & 1 (all four warps, one row each)
  auto epilogue = [&](int j) {
    float best_v = __int_as_float(0x7F800000);
    int best = 0;
    for (int cc = 0; cc < Cp / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)((j & 1) * Cp + cc * 32), v);
      tmem_wait_ld();
      #pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int n = cc * 32 + i;
        const float sc = sbias[n] - 2.f * __uint_as_float(v[i]);
        if (n < C && sc < best_v) { best_v = sc; best = n; }
      }
    }
    const int t = m_base + j * kAsgRows + warp * 32 + lane;
    const int lab = t < s.n_pad ? (token_valid(s, t) ? best : C) : -1;
    if (lab >= 0) labels[(size_t)bh * s.n_pad + t] = lab;
    // one shared-memory atomic per distinct label of the warp
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, lab);
    if (lab >= 0 && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[lab], __popc(peers));
  };

  for (int i = 0; i <= tiles; ++i) {
    if (*abort_flag) break;                 // uniform: read after the barrier that ends each pass
    if (i < tiles && threadIdx.x == 0) {
      bool ok = (i > 0 || mbar_wait(u_full, 0, abort_flag, status)) &&
                mbar_wait(&x_full[i % nst], (uint32_t)(i / nst) & 1u, abort_flag, status);
      if (ok) {
        ++landed;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)((i & 1) * Cp);
        uint32_t acc = 0;
        #pragma unroll
        for (int part = 0; part < 3; ++part) {
          #pragma unroll
          for (int c = 0; c < L::kAChunks; ++c) {
            const uint32_t a = smem_u32(sX + (i % nst) * L::kXBytes + c * L::kAChunkBytes);
            const uint32_t b = smem_u32(sU + (part * L::kAChunks + c) * b_chunk);
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_bf16_ss(d, desc_kmajor(a + kk * 32), desc_kmajor(b + kk * 32), id, acc);
              acc = 1;
            }
          }
        }
        mma_commit(&mma_done[i & 1]);
        // the stage of tile i - 1 is free once its MMAs are done: load tile i + nst - 1 into it
        if (i + nst - 1 < tiles &&
            (i == 0 || mbar_wait(&mma_done[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, abort_flag, status)))
          load_x(i + nst - 1);
      }
    }
    if (i > 0) {
      const int j = i - 1;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&mma_done[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag,
                                                        status));
      tc_fence_after();
      if (ok) epilogue(j);
    }
    tc_fence_before();
    __syncthreads();                        // TMEM buffer (i - 1) & 1 is read before tile i + 1 reuses it
    tc_fence_after();
  }
  if (threadIdx.x == 0) {
    // loads still in flight land before the shared memory is released; the MMAs issued
    // so far are done before TMEM is released
    for (int i = landed; i < issued; ++i) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&x_full[i % nst], (uint32_t)(i / nst) & 1u) &&
             clock64() - t0 < kWaitBudgetCycles) {}
    }
    mma_commit(drain);
  }
  {
    const long long t0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
  }
  tc_fence_after();
  __syncthreads();
  if (!*abort_flag) {
    int32_t* cnt = counts + ((size_t)bh * n_chunks + chunk) * (C + 1);
    for (int i = threadIdx.x; i <= C; i += blockDim.x)
      if (hist[i]) atomicAdd(&cnt[i], hist[i]);
  }
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, (uint32_t)(2 * Cp)); }
}

// ------------------------------------------------------------------ counting sort
// Exclusive offsets of every (chunk, bucket): the tokens of bucket b in chunk ch start at
// offs[ch][b] = start[b] + (tokens of bucket b in chunks before ch).  The counts are
// cleared on the way, ready for the next step's histogram.  Also the piece offsets of the
// centre update: cluster n (< C) is cut into ceil(size / kPiece) pieces of consecutive
// positions, the first of which is piece poff[n]; poff[C] = the number of pieces.
constexpr int kPiece = 256;
__global__ void __launch_bounds__(256) svoo_scan_kernel(int32_t* __restrict__ counts, int32_t* __restrict__ offs,
                                                        int32_t* __restrict__ start, int32_t* __restrict__ poff,
                                                        int n_chunks, int C) {
  __shared__ int total[kHistSlots];
  __shared__ int base[kHistSlots + 1];
  const int bh = blockIdx.x, b = threadIdx.x, nbk = C + 1;
  int32_t* cnt = counts + (size_t)bh * n_chunks * nbk;
  int32_t* off = offs + (size_t)bh * n_chunks * nbk;
  if (b < nbk) {
    int run = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 8) {
      int v[8];
      #pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = c0 + j < n_chunks ? cnt[(size_t)(c0 + j) * nbk + b] : 0;
      #pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (c0 + j < n_chunks) {
          off[(size_t)(c0 + j) * nbk + b] = run;
          cnt[(size_t)(c0 + j) * nbk + b] = 0;
        }
        run += v[j];
      }
    }
    total[b] = run;
  }
  __syncthreads();
  if (b == 0) {
    int r = 0, pr = 0;
    for (int i = 0; i < nbk; ++i) { base[i] = r; r += total[i]; }
    base[nbk] = r;
    for (int i = 0; i < C; ++i) { poff[(size_t)bh * (C + 1) + i] = pr; pr += (total[i] + kPiece - 1) / kPiece; }
    poff[(size_t)bh * (C + 1) + C] = pr;
  }
  __syncthreads();
  if (b < nbk)
    for (int ch = 0; ch < n_chunks; ++ch) off[(size_t)ch * nbk + b] += base[b];
  if (b <= nbk) start[(size_t)bh * (C + 2) + b] = base[b];
}

// perm[offs[ch][label] + (earlier tokens of the chunk with that label)] = token, for the
// tokens of one chunk taken in index order, 256 at a time: within a warp the rank comes
// from __match_any_sync, across warps from the per-warp label counts.
__global__ void __launch_bounds__(kScatterThreads) svoo_scatter_kernel(const int32_t* __restrict__ labels,
                                                                       const int32_t* __restrict__ offs,
                                                                       int32_t* __restrict__ perm, int n_chunks,
                                                                       int C, int n_pad) {
  constexpr int kWarps = kScatterThreads / 32;
  __shared__ int run[kHistSlots];
  __shared__ int wcnt[kWarps][kHistSlots];
  const int ch = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbk = C + 1;
  for (int i = tid; i < nbk; i += kScatterThreads) run[i] = offs[((size_t)bh * n_chunks + ch) * nbk + i];
  for (int i = tid; i < kWarps * kHistSlots; i += kScatterThreads) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  for (int it = 0; it < kSortChunk / kScatterThreads; ++it) {
    const int t = ch * kSortChunk + it * kScatterThreads + tid;
    int lab = t < n_pad ? labels[(size_t)bh * n_pad + t] : -1;
    if (lab > C) lab = -1;                  // never from a completed assignment (its status is set)
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, lab);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (lab >= 0 && rank == 0) wcnt[warp][lab] = __popc(peers);
    __syncthreads();
    if (lab >= 0) {
      int pos = run[lab] + rank;
      for (int w = 0; w < warp; ++w) pos += wcnt[w][lab];
      if (pos >= 0 && pos < n_pad) perm[(size_t)bh * n_pad + pos] = t;
    }
    __syncthreads();
    for (int i = tid; i < nbk; i += kScatterThreads) {
      int sum = 0;
      #pragma unroll
      for (int w = 0; w < kWarps; ++w) { sum += wcnt[w][i]; wcnt[w][i] = 0; }
      run[i] += sum;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ centre update
// Centre n = mean of the tokens at positions [start[n], start[n+1]) of the order, in fp64,
// in two deterministic passes.  svoo_piece_kernel: one CTA per piece of kPiece consecutive
// positions of one cluster (their token indices staged in shared memory); warp w sums rows
// w, w + 8, ... of the piece, lane l owning channels [l D/32, (l+1) D/32), and the eight warp
// sums are added in warp order into part[piece].  svoo_finalize_kernel: the pieces of each
// cluster are added in order and divided by its size; an empty cluster keeps its centre.
template <int D>
__global__ void __launch_bounds__(256) svoo_piece_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const int32_t* __restrict__ perm,
                                                         const int32_t* __restrict__ start,
                                                         const int32_t* __restrict__ poff,
                                                         double* __restrict__ part, int C, int n_pad,
                                                         int max_pieces) {
  constexpr int kPer = D / 32;              // channels per lane: 4 (d = 128) or 2 (d = 64)
  __shared__ int sp[kPiece];
  __shared__ double red[8][D];
  __shared__ int s_n;
  const int p = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t* po = poff + (size_t)bh * (C + 1);
  if (p >= po[C]) return;                   // uniform: fewer pieces than the bound
  if (tid == 0) {                           // the cluster of this piece: the last n with poff[n] <= p
    int lo = 0, hi = C - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (po[mid] <= p) lo = mid; else hi = mid - 1;
    }
    s_n = lo;
  }
  __syncthreads();
  const int n = s_n;
  const int p0 = start[(size_t)bh * (C + 2) + n] + (p - po[n]) * kPiece;
  const int p1 = min(start[(size_t)bh * (C + 2) + n + 1], p0 + kPiece);
  const int cnt = p1 - p0;
  if (tid < cnt) sp[tid] = perm[(size_t)bh * n_pad + p0 + tid];
  __syncthreads();
  const __nv_bfloat16* xb = x + (size_t)bh * n_pad * D;
  double acc[kPer];
  #pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.0;
  #pragma unroll 8
  for (int j = warp; j < cnt; j += 8) {
    const int t = sp[j];
    if ((unsigned)t >= (unsigned)n_pad) continue;     // only after an aborted assignment
    const __nv_bfloat16* row = xb + (size_t)t * D + lane * kPer;
    if constexpr (kPer == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(row);
      acc[0] += (double)bf16_lo(w.x); acc[1] += (double)bf16_hi(w.x);
      acc[2] += (double)bf16_lo(w.y); acc[3] += (double)bf16_hi(w.y);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row);
      acc[0] += (double)bf16_lo(w); acc[1] += (double)bf16_hi(w);
    }
  }
  #pragma unroll
  for (int i = 0; i < kPer; ++i) red[warp][lane * kPer + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    double sum = 0.0;
    #pragma unroll
    for (int w = 0; w < 8; ++w) sum += red[w][tid];
    part[((size_t)bh * max_pieces + p) * D + tid] = sum;
  }
}

__global__ void svoo_finalize_kernel(const double* __restrict__ part, const int32_t* __restrict__ start,
                                     const int32_t* __restrict__ poff, float* __restrict__ centres, int C, int Cp,
                                     int d, int max_pieces) {
  const int n = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const int size = start[(size_t)bh * (C + 2) + n + 1] - start[(size_t)bh * (C + 2) + n];
  if (size <= 0) return;
  const int q0 = poff[(size_t)bh * (C + 1) + n], q1 = poff[(size_t)bh * (C + 1) + n + 1];
  double sum = 0.0;
  for (int q = q0; q < q1; ++q) sum += part[((size_t)bh * max_pieces + q) * d + c];
  centres[((size_t)bh * Cp + n) * d + c] = (float)(sum / (double)size);
}

// ------------------------------------------------------------------ row gather / scatter
// A row of D bf16 moves as D/8 16-byte pieces; a warp moves 32 / (D/8) rows at a time.
// gather:  dst_i[p] = src_i[perm_i[p]] for the three tensors (q with q_perm, k and v with
//          k_perm); scatter: out[q_perm[p]] = src[p].  An index outside [0, n_pad) sets
//          SLR_ERR_INDEX in the status word; the gather then writes zeros, the scatter skips.
template <int D>
__global__ void __launch_bounds__(256) svoo_gather_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                          const uint4* __restrict__ v,
                                                          const int32_t* __restrict__ q_perm,
                                                          const int32_t* __restrict__ k_perm, uint4* __restrict__ qp,
                                                          uint4* __restrict__ kp, uint4* __restrict__ vp,
                                                          long long rows, int n_pad, int* status) {
  constexpr int kPieces = D / 8;
  constexpr int kGroups = 32 / kPieces;
  const int lane = threadIdx.x & 31, g = lane / kPieces, li = lane % kPieces;
  const long long units = rows * 3;
  const long long stride = (long long)gridDim.x * (blockDim.x >> 5) * kGroups;
  for (long long u = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kGroups + g; u < units;
       u += stride) {
    const long long r = u / 3;
    const int which = (int)(u - r * 3);
    const long long base = r - r % n_pad;   // first row of this (b, h)
    const int t = which == 0 ? q_perm[r] : k_perm[r];
    const uint4* src = which == 0 ? q : (which == 1 ? k : v);
    uint4* dst = which == 0 ? qp : (which == 1 ? kp : vp);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0 && t < n_pad) {
      val = src[(base + t) * kPieces + li];
    } else if (li == 0) {
      atomicCAS(status, 0, kErrIndex);
    }
    dst[r * kPieces + li] = val;
  }
}

template <int D>
__global__ void __launch_bounds__(256) svoo_scatter_rows_kernel(const uint4* __restrict__ src,
                                                                const int32_t* __restrict__ q_perm,
                                                                uint4* __restrict__ out, long long rows, int n_pad,
                                                                int* status) {
  constexpr int kPieces = D / 8;
  constexpr int kGroups = 32 / kPieces;
  const int lane = threadIdx.x & 31, g = lane / kPieces, li = lane % kPieces;
  const long long stride = (long long)gridDim.x * (blockDim.x >> 5) * kGroups;
  for (long long r = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kGroups + g; r < rows;
       r += stride) {
    const int t = q_perm[r];
    if (t >= 0 && t < n_pad) {
      out[(r - r % n_pad + t) * kPieces + li] = src[r * kPieces + li];
    } else if (li == 0) {
      atomicCAS(status, 0, kErrIndex);
    }
  }
}

// Blocks of 8 warps for `warp_tasks` warp-sized pieces of work, at most 16 blocks per SM
// (the loops stride over the rest).
int copy_grid(long long warp_tasks) {
  long long blocks = (warp_tasks + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

// ------------------------------------------------------------------ launchers

int svoo_padded_clusters(int C) {
  int cp = 32;
  while (cp < C) cp *= 2;
  return cp;
}

int svoo_sort_chunks(int n_pad) { return (n_pad + kSortChunk - 1) / kSortChunk; }

cudaError_t launch_svoo_anchors(const void* x, const int32_t* anchor, float* centres, int C, int BH, int d,
                                SeqShape s, int* status, cudaStream_t st) {
  const int Cp = svoo_padded_clusters(C);
  svoo_anchor_kernel<<<dim3(Cp, BH), d, 0, st>>>(static_cast<const __nv_bfloat16*>(x), anchor, centres, C, Cp, d,
                                                  s, status);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_assign_d(const void* x, const __nv_bfloat16* ub, const float* bias, int C, int Cp,
                            int32_t* labels, int32_t* counts, int BH, SeqShape s, int* status, cudaStream_t st) {
  using L = AsgLayout<D>;
  CUtensorMap mx, mu;
  const uint64_t xd[3] = {(uint64_t)D, (uint64_t)s.n_pad, (uint64_t)BH};
  const uint64_t xs[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * s.n_pad};
  const uint32_t xb[3] = {64, kAsgRows, 1};
  if (!make_tile_map(&mx, x, 3, xd, xs, xb)) return cudaErrorInvalidValue;
  const uint64_t ud[3] = {(uint64_t)(3 * D), (uint64_t)Cp, (uint64_t)BH};
  const uint64_t us[2] = {(uint64_t)(3 * D) * 2, (uint64_t)(3 * D) * 2 * Cp};
  const uint32_t ubx[3] = {64, (uint32_t)Cp, 1};
  if (!make_tile_map(&mu, ub, 3, ud, us, ubx)) return cudaErrorInvalidValue;
  const int nst = L::stages(Cp);
  const size_t smem = L::bytes(Cp, nst);
  cudaError_t e = cudaFuncSetAttribute(svoo_assign_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(svoo_sort_chunks(s.n_pad), BH);
  svoo_assign_kernel<D><<<grid, 128, smem, st>>>(mx, mu, bias, C, Cp, labels, counts, svoo_sort_chunks(s.n_pad), s,
                                                 nst, status);
  return cudaGetLastError();
}

cudaError_t launch_svoo_assign(const void* x, const float* other, int C_other, float* own, int C_own,
                               __nv_bfloat16* ub, float* bias, int32_t* labels, int32_t* counts, int BH, int d,
                               SeqShape s, int* status, cudaStream_t st) {
  const int Cpo = svoo_padded_clusters(C_other), Cp = svoo_padded_clusters(C_own);
  const int msmem = C_other * d * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(svoo_metric_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem);
  if (e != cudaSuccess) return e;
  svoo_metric_kernel<<<dim3(Cp, BH), 128, msmem, st>>>(other, C_other, Cpo, own, C_own, Cp, d, ub, bias);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return d == 128 ? launch_assign_d<128>(x, ub, bias, C_own, Cp, labels, counts, BH, s, status, st)
                  : launch_assign_d<64>(x, ub, bias, C_own, Cp, labels, counts, BH, s, status, st);
}

cudaError_t launch_svoo_sort(const int32_t* labels, int32_t* counts, int32_t* offs, int32_t* start, int32_t* poff,
                             int32_t* perm, int C, int BH, SeqShape s, cudaStream_t st) {
  const int nch = svoo_sort_chunks(s.n_pad);
  svoo_scan_kernel<<<BH, 256, 0, st>>>(counts, offs, start, poff, nch, C);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  svoo_scatter_kernel<<<dim3(nch, BH), kScatterThreads, 0, st>>>(labels, offs, perm, nch, C, s.n_pad);
  return cudaGetLastError();
}

int svoo_max_pieces(int n_pad, int C) { return (n_pad + kPiece - 1) / kPiece + C; }

cudaError_t launch_svoo_update(const void* x, const int32_t* perm, const int32_t* start, const int32_t* poff,
                               double* part, float* centres, int C, int BH, int d, SeqShape s, cudaStream_t st) {
  const int Cp = svoo_padded_clusters(C);
  const int mp = svoo_max_pieces(s.n_pad, C);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (d == 128)
    svoo_piece_kernel<128><<<dim3(mp, BH), 256, 0, st>>>(xb, perm, start, poff, part, C, s.n_pad, mp);
  else
    svoo_piece_kernel<64><<<dim3(mp, BH), 256, 0, st>>>(xb, perm, start, poff, part, C, s.n_pad, mp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  svoo_finalize_kernel<<<dim3(C, BH), d, 0, st>>>(part, start, poff, centres, C, Cp, d, mp);
  return cudaGetLastError();
}

cudaError_t launch_svoo_gather(const void* q, const void* k, const void* v, const int32_t* q_perm,
                               const int32_t* k_perm, void* qp, void* kp, void* vp, int BH, int d, int n_pad,
                               int* status, cudaStream_t st) {
  const long long rows = (long long)BH * n_pad;
  const uint4* a = static_cast<const uint4*>(q);
  const uint4* b = static_cast<const uint4*>(k);
  const uint4* c = static_cast<const uint4*>(v);
  uint4* x = static_cast<uint4*>(qp);
  uint4* y = static_cast<uint4*>(kp);
  uint4* z = static_cast<uint4*>(vp);
  if (d == 128)
    svoo_gather_kernel<128><<<copy_grid(rows * 3 / 2), 256, 0, st>>>(a, b, c, q_perm, k_perm, x, y, z, rows, n_pad,
                                                                      status);
  else
    svoo_gather_kernel<64><<<copy_grid(rows * 3 / 4), 256, 0, st>>>(a, b, c, q_perm, k_perm, x, y, z, rows, n_pad,
                                                                     status);
  return cudaGetLastError();
}

cudaError_t launch_svoo_scatter_rows(const void* src, const int32_t* q_perm, void* out, int BH, int d, int n_pad,
                                     int* status, cudaStream_t st) {
  const long long rows = (long long)BH * n_pad;
  const uint4* a = static_cast<const uint4*>(src);
  uint4* o = static_cast<uint4*>(out);
  if (d == 128)
    svoo_scatter_rows_kernel<128><<<copy_grid(rows / 2), 256, 0, st>>>(a, q_perm, o, rows, n_pad, status);
  else
    svoo_scatter_rows_kernel<64><<<copy_grid(rows / 4), 256, 0, st>>>(a, q_perm, o, rows, n_pad, status);
  return cudaGetLastError();
}

}  // namespace slr
