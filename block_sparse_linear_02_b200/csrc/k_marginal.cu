// k_marginal.cu -- the linear-attention branch of SLA on tcgen05 (sm_100a).
//
// SLA page section 3 (the marginal-weight branch): for marginal block pairs the
// attention is replaced by linear attention with feature map phi, evaluated by
// forming K^T V first and applying Q afterwards; its output passes through the learnable
// projection W_proj before it is added (same section, projection paragraph).
// Because linear attention is a normalised weighted sum of value rows,
// (sum w v / sum w) W = sum w (v W) / sum w, so W_proj is folded into V here.
//
//  key_states_kernel    persistent over key blocks; per block j: (V_j W)^T by one MMA (M=128 channels,
//                       N=64 tokens, K=d), then h_j'^T = (V_j W)^T phi(K_j)
//                       (M=128, N=d, K=64 tokens; phi applied in place in shared
//                       memory) and z_j = sum_t phi(K_j,t); written as bf16 rows
//                       [h_j'^T ; z_j] of (d+1)*d elements.  Without W the first
//                       MMA is skipped and V_j^T is read MN-major from the tile.
//  reduce_states_kernel per head: Hs = M01 . h, a persistent tensor-core GEMM
//                       with the 0/1 marginal indicator M01 [Nqb x Nkb]
//                       (K-major) and h [Nkb x (d+1)d] (MN-major), fp32
//                       accumulation in two TMEM buffers, bf16 out.  Row i of
//                       Hs is [H_i'^T ; Z_i].
//  linear_apply_kernel  per pair of query blocks: phi(Q) times the rows
//                       [H_i'^T ; Z_i] (M=128 tokens, N=d+16), whose column d is
//                       the denominator phi(q_t).Z_i; fp32 [token][channel] out.
//                       (The SLA call does this step inside the attention
//                       kernel's epilogue instead.)
// d = 64 runs the same M=128 MMAs with the upper 64 rows of A zero-filled.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Block-wide bounded wait: every thread polls; any timeout aborts all.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort, status));
}

// ------------------------------------------------------------------ key states
// Persistent: each CTA walks key blocks b = blockIdx.x, blockIdx.x + gridDim.x, ...
// with a 2-stage TMA ring (the next block's K/V load overlaps this block's work)
// and W_proj loaded once.  Shared memory (bytes): W 32K | 2 x (K 16K, V 16K) | z 4K.
// (V W)^T is written back over the V stage it was computed from.
constexpr int kKsW = 0, kKsRing = 32768, kKsStage = 32768, kKsZ = kKsRing + 2 * kKsStage;
constexpr int kKsBar = kKsZ + 4096;
constexpr int kKsSmem = kKsBar + 128 + 1024;

template <int D, bool PROJ>
__global__ void __launch_bounds__(128, 2)
key_states_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmW, __nv_bfloat16* __restrict__ h, SeqShape s, int BH,
                  int phi, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem + kKsW;               // W_proj MN-major: rows c_in, 64 c_out per chunk (chunk stride D*128)
  float* zred = reinterpret_cast<float*>(smem + kKsZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kKsBar);
  uint64_t* load = bars;                   // [2]
  uint64_t* w_bar = bars + 2;
  uint64_t* mma0 = bars + 3;
  uint64_t* mma1 = bars + 4;
  uint64_t* drain = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr uint32_t kColP = 0;            // (V W)^T: 64 columns
  constexpr uint32_t kColH = 64;           // h^T: D columns
  constexpr int kChunkB = 8192;            // one 64-row x 128-byte chunk
  const int total = BH * s.n_blocks;
  auto sK = [&](int st) { return smem + kKsRing + st * kKsStage; };
  auto sV = [&](int st) { return smem + kKsRing + st * kKsStage + 16384; };

  if (tid == 0) {
    mbar_init(&load[0], 1);
    mbar_init(&load[1], 1);
    mbar_init(w_bar, 1);
    mbar_init(mma0, 1);
    mbar_init(mma1, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (D == 64) {
    // upper half of the M = 128 A operand must be zero (W chunk 1, or V's second 8 KB)
    for (int i = tid; i < 8192 / 16; i += 128) {
      if (PROJ) reinterpret_cast<uint4*>(sW + D * 128)[i] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sV(0) + 8192)[i] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sV(1) + 8192)[i] = make_uint4(0, 0, 0, 0);
    }
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto issue_load = [&](int n, int st) {
    const int blk_id = blockIdx.x + n * gridDim.x;
    const int bh = blk_id / s.n_blocks, blk = blk_id % s.n_blocks;
    mbar_arrive_expect_tx(&load[st], 2 * (D / 64) * kChunkB);
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sK(st) + c * kChunkB, &tmK, &load[st], c * 64, blk * 64, bh);
      tma_load_3d(sV(st) + c * kChunkB, &tmV, &load[st], c * 64, blk * 64, bh);
    }
  };
  const int mine = blockIdx.x < total ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (tid == 0 && mine > 0) {
    if (PROJ) {
      mbar_arrive_expect_tx(w_bar, (D / 64) * D * 128);
      for (int c = 0; c < D / 64; ++c) tma_load_3d(sW + c * D * 128, &tmW, w_bar, c * 64, 0, 0);
    }
    issue_load(0, 0);
    if (mine > 1) issue_load(1, 1);
  }
  bool ok = true;
  if (PROJ && mine > 0) ok = cta_wait(w_bar, 0, abort_flag, status);

  constexpr int kCPR = D / 8, kRS = 128 / kCPR;
  const int g = tid % kCPR, rs = tid / kCPR;
  const int chunk = g >> 3, q8 = g & 7;
  for (int n = 0; n < mine && ok; ++n) {
    const int st = n & 1;
    const int blk_id = blockIdx.x + n * gridDim.x;
    const int bh = blk_id / s.n_blocks, blk = blk_id % s.n_blocks;
    uint8_t* k_s = sK(st);
    uint8_t* v_s = sV(st);
    if (!(ok = cta_wait(&load[st], (n >> 1) & 1, abort_flag, status))) break;
    if (PROJ && tid == 0) {
      // (V_j W)^T = W^T V_j^T: M = c_out (128), N = t (64), K = c_in (D)
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16(128, 64, true, false);
      #pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = desc_mnmajor(smem_u32(sW) + kk * 2048, D * 128);
        const uint64_t b = desc_kmajor(smem_u32(v_s) + (kk >> 2) * kChunkB + (kk & 3) * 32);
        mma_bf16_ss(tmem + kColP, a, b, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(mma0);
    }
    // phi in place (pad tokens -> 0) and column sums z
    const int nvalid = block_valid_count(s, blk);
    float z[8];
    #pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = 0.f;
    for (int t = rs; t < 64; t += kRS) {       // the same trip count in every lane
      uint4* pk = reinterpret_cast<uint4*>(k_s + chunk * kChunkB + sw128_offset(t, q8));
      const uint4 u = *pk;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      float f[8];
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
      }
      if (phi == SLR_PHI_SOFTMAX) {
        row_softmax8<kCPR>(f);                 // the kCPR lanes of row t
      } else {
        #pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = phi_elu1(f[i]);
      }
      uint32_t o[4];
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = t < nvalid ? f[2 * i] : 0.f;
        const float b = t < nvalid ? f[2 * i + 1] : 0.f;
        z[2 * i] += a;
        z[2 * i + 1] += b;
        o[i] = pack_bf16(a, b);
      }
      *pk = make_uint4(o[0], o[1], o[2], o[3]);
    }
    #pragma unroll
    for (int i = 0; i < 8; ++i) zred[rs * D + g * 8 + i] = z[i];
    if (PROJ) {
      // (V W)^T from TMEM over the V stage (V has been consumed): K-major A of the next MMA
      if (!(ok = cta_wait(mma0, n & 1, abort_flag, status))) break;
      tc_fence_after();
      uint32_t r[32], r2[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kColP, r);
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kColP + 32, r2);
      tmem_wait_ld();
      #pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint32_t* src = c8 < 4 ? r : r2;
        const int b = (c8 & 3) * 8;
        *reinterpret_cast<uint4*>(v_s + sw128_offset(tid, c8)) =
            make_uint4(pack_bf16(__uint_as_float(src[b]), __uint_as_float(src[b + 1])),
                       pack_bf16(__uint_as_float(src[b + 2]), __uint_as_float(src[b + 3])),
                       pack_bf16(__uint_as_float(src[b + 4]), __uint_as_float(src[b + 5])),
                       pack_bf16(__uint_as_float(src[b + 6]), __uint_as_float(src[b + 7])));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      // h^T: M = c (128), N = a (D), K = t (64)
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16(128, D, !PROJ, true);
      #pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = PROJ ? desc_kmajor(smem_u32(v_s) + kk * 32) : desc_mnmajor(smem_u32(v_s) + kk * 2048, kChunkB);
        const uint64_t b = desc_mnmajor(smem_u32(k_s) + kk * 2048, kChunkB);
        mma_bf16_ss(tmem + kColH, a, b, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(mma1);
    }
    __nv_bfloat16* hrow = h + ((size_t)bh * s.n_blocks + blk) * (size_t)(D + 1) * D;
    for (int a = tid; a < D; a += 128) {
      float sum = 0.f;
      #pragma unroll
      for (int r = 0; r < kRS; ++r) sum += zred[r * D + a];
      hrow[(size_t)D * D + a] = __float2bfloat16_rn(sum);
    }
    if (!(ok = cta_wait(mma1, n & 1, abort_flag, status))) break;
    tc_fence_after();
    if (warp * 32 < D) {
      const int c = tid;                     // TMEM lane = output row (value channel)
      #pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kColH + cc * 32, r);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(hrow + (size_t)c * D + cc * 32);
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pack_bf16(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                              pack_bf16(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                              pack_bf16(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                              pack_bf16(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
      }
    }
    tc_fence_before();
    __syncthreads();                          // stage st and the TMEM results are no longer read
    if (tid == 0 && n + 2 < mine) issue_load(n + 2, st);
  }
  if (!ok && tid == 0) {
    mma_commit(drain);
    const long long t0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 256); }
}

// ------------------------------------------------------------------ key states, d = 128
// Warp-specialised and persistent (one CTA per SM, 448 threads): warp 0 streams K_j,
// V_j into a 3-stage ring; warp 1 issues the MMAs; warps 2-9 apply phi in place and
// form z_j, warps 2-5 also move (V_j W)^T from TMEM into the operand layout of the
// second MMA; warps 10-13 drain h_j'^T from TMEM into a swizzled staging tile that two
// TMA stores write out.
// TMEM holds two (V W)^T and two h^T accumulators, so block n's drain overlaps block
// n+1's phi and MMAs.  Every hand-off goes through an mbarrier with a bounded wait.
constexpr int kKpStages = 3;
struct KpLayout {
  static constexpr int kW = 0;                               // W_proj MN-major, 2 chunks x 16 KB
  static constexpr int kRing = 32768;                        // stages: K 16 KB | V 16 KB
  static constexpr int kStage = 32768;
  static constexpr int kOut = kRing + kKpStages * kStage;    // h^T staging: 2 boxes of 64 columns
  static constexpr int kZ = kOut + 32768;                    // z partials [2][16][128] floats
  static constexpr int kBar = kZ + 2 * 16 * 128 * 4;
  static constexpr int kBytes = kBar + 256 + 1024;
};

__device__ __forceinline__ float phi_exp2(float x) {
  // elu(x) + 1 = exp(min(x, 0)) + max(x, 0), branch-free; exp through the exp2 unit
  // (the result is rounded to bf16)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fminf(x, 0.f) * 1.4426950408889634f));
  return y + fmaxf(x, 0.f);
}


template <bool PROJ>
__global__ void __launch_bounds__(448, 1)
key_states_pipe_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmH,
                       __nv_bfloat16* __restrict__ h, SeqShape s, int BH, int phi, int* status) {
  constexpr int D = 128;
  using L = KpLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem + L::kW;
  uint8_t* sOut = smem + L::kOut;
  float* zbuf = reinterpret_cast<float*>(smem + L::kZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* full = bars;                          // [3] stage loaded
  uint64_t* empty = full + kKpStages;             // [3] stage consumed by the second MMA
  uint64_t* w_bar = empty + kKpStages;
  uint64_t* p_full = w_bar + 1;                   // [2] (V W)^T in TMEM
  uint64_t* conv_done = p_full + 2;               // [2] operands of the second MMA ready (256 arrivals)
  uint64_t* h_full = conv_done + 2;               // [2] h^T in TMEM
  uint64_t* h_free = h_full + 2;                  // [2] h^T drained (128 arrivals)
  uint64_t* out_free = h_free + 2;                // staging tile read by the previous stores
  uint64_t* out_full = out_free + 1;              // staging tile written (128 arrivals)
  uint64_t* z_ready = out_full + 1;               // [2] z partials of a block written (256 arrivals)
  uint64_t* drain = z_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kChunkB = 8192;                   // 64 rows x 128 bytes
  constexpr uint32_t kColP = 0;                   // P[b] at b * 64
  constexpr uint32_t kColH = 128;                 // H[b] at 128 + b * 128
  const int total = BH * s.n_blocks;
  const int mine = blockIdx.x < total ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto sK = [&](int st) { return smem + L::kRing + st * L::kStage; };
  auto sV = [&](int st) { return smem + L::kRing + st * L::kStage + 16384; };

  if (tid == 0) {
    for (int i = 0; i < kKpStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(w_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&p_full[b], 1);
      mbar_init(&conv_done[b], 256);
      mbar_init(&h_full[b], 1);
      mbar_init(&h_free[b], 128);
    }
    mbar_init(out_free, 1);
    mbar_init(out_full, 128);
    mbar_init(&z_ready[0], 256);
    mbar_init(&z_ready[1], 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && mine > 0) {
      tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      if (PROJ) {
        mbar_arrive_expect_tx(w_bar, 2 * D * 128);
        for (int c = 0; c < 2; ++c) tma_load_3d(sW + c * D * 128, &tmW, w_bar, c * 64, 0, 0);
      }
      int n = 0;
      for (; n < mine; ++n) {
        const int st = n % kKpStages;
        if (n >= kKpStages && !mbar_wait(&empty[st], ((n / kKpStages) - 1) & 1, abort_flag, status)) break;
        const int blk_id = blockIdx.x + n * gridDim.x;
        const int bh = blk_id / s.n_blocks, blk = blk_id % s.n_blocks;
        mbar_arrive_expect_tx(&full[st], 2 * 2 * kChunkB);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sK(st) + c * kChunkB, &tmK, &full[st], c * 64, blk * 64, bh);
          tma_load_3d(sV(st) + c * kChunkB, &tmV, &full[st], c * 64, blk * 64, bh);
        }
      }
      if (*abort_flag) {
        long long t0 = clock64();
        if (PROJ) while (!mbar_try_wait(w_bar, 0) && clock64() - t0 < kWaitBudgetCycles) {}
        for (int i = (n - kKpStages > 0 ? n - kKpStages : 0); i < n; ++i) {
          t0 = clock64();
          while (!mbar_try_wait(&full[i % kKpStages], (i / kKpStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && mine > 0) {
      bool ok = !PROJ || mbar_wait(w_bar, 0, abort_flag, status);
      for (int n = 0; n < mine && ok; ++n) {
        const int st = n % kKpStages, b = n & 1;
        if (!(ok = mbar_wait(&full[st], (n / kKpStages) & 1, abort_flag, status))) break;
        tc_fence_after();
        if (PROJ) {
          // (V_j W)^T = W^T V_j^T: M = c_out, N = t (64), K = c_in
          constexpr uint32_t id = idesc_bf16(128, 64, true, false);
          #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = desc_mnmajor(smem_u32(sW) + kk * 2048, D * 128);
            const uint64_t bd = desc_kmajor(smem_u32(sV(st)) + (kk >> 2) * kChunkB + (kk & 3) * 32);
            mma_bf16_ss(tmem + kColP + b * 64, a, bd, id, kk > 0 ? 1u : 0u);
          }
          mma_commit(&p_full[b]);
        }
        if (!(ok = mbar_wait(&conv_done[b], (n >> 1) & 1, abort_flag, status))) break;
        if (n >= 2 && !(ok = mbar_wait(&h_free[b], ((n - 2) >> 1) & 1, abort_flag, status))) break;
        tc_fence_after();
        // h^T: M = c (value channel), N = a (key feature), K = t (64 tokens)
        constexpr uint32_t id = idesc_bf16(128, D, !PROJ, true);
        #pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = PROJ ? desc_kmajor(smem_u32(sV(st)) + kk * 32)
                                  : desc_mnmajor(smem_u32(sV(st)) + kk * 2048, kChunkB);
          const uint64_t bd = desc_mnmajor(smem_u32(sK(st)) + kk * 2048, kChunkB);
          mma_bf16_ss(tmem + kColH + b * 128, a, bd, id, kk > 0 ? 1u : 0u);
        }
        mma_commit(&h_full[b]);
        mma_commit(&empty[st]);
      }
      if (!ok) {
        mma_commit(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- phi warps
    const int pt = tid - 64;                       // 0..255
    const bool conv = warp < 6;                    // warps 2-5 also move (V W)^T
    const int c = (warp & 3) * 32 + lane;          // my TMEM lane = row of (V W)^T
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    constexpr int kCPR = D / 8, kRS = 256 / kCPR;  // 16 chunks of 8 channels, 16 row sets
    const int g = pt % kCPR, rs = pt / kCPR;
    const int chunk = g >> 3, q8 = g & 7;
    bool ok = true;
    for (int n = 0; n < mine && ok; ++n) {
      const int st = n % kKpStages, b = n & 1;
      const int blk_id = blockIdx.x + n * gridDim.x;
      const int bh = blk_id / s.n_blocks, blk = blk_id % s.n_blocks;
      if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[st], (n / kKpStages) & 1, abort_flag, status)))) break;
      // phi in place (pad tokens -> 0) and partial column sums
      const int nvalid = block_valid_count(s, blk);
      float z[8];
      #pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = 0.f;
      uint8_t* k_s = sK(st);
      #pragma unroll
      for (int tt = 0; tt < 64 / kRS; ++tt) {
        const int t = rs + tt * kRS;
        uint4* pk = reinterpret_cast<uint4*>(k_s + chunk * kChunkB + sw128_offset(t, q8));
        const uint4 u = *pk;
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        float f[8];
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          f[2 * i] = bf16_lo(w[i]);
          f[2 * i + 1] = bf16_hi(w[i]);
        }
        if (phi == SLR_PHI_SOFTMAX) {
          row_softmax8<kCPR>(f);               // the kCPR lanes of row t (a half warp)
        } else {
          #pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = phi_exp2(f[i]);
        }
        uint32_t o[4];
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x0 = t < nvalid ? f[2 * i] : 0.f;
          const float x1 = t < nvalid ? f[2 * i + 1] : 0.f;
          z[2 * i] += x0;
          z[2 * i + 1] += x1;
          o[i] = pack_bf16(x0, x1);
        }
        *pk = make_uint4(o[0], o[1], o[2], o[3]);
      }
      #pragma unroll
      for (int i = 0; i < 8; ++i) zbuf[(b * kRS + rs) * D + g * 8 + i] = z[i];
      mbar_arrive(&z_ready[b]);
      if (PROJ && conv) {
        // (V W)^T from TMEM over the V stage (V has been consumed): K-major A operand
        if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&p_full[b], (n >> 1) & 1, abort_flag, status)))) break;
        tc_fence_after();
        uint32_t r[32], r2[32];
        tmem_ld32(lane_addr + kColP + b * 64, r);
        tmem_ld32(lane_addr + kColP + b * 64 + 32, r2);
        tmem_wait_ld();
        uint8_t* v_s = sV(st);
        #pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint32_t* src = c8 < 4 ? r : r2;
          const int o = (c8 & 3) * 8;
          *reinterpret_cast<uint4*>(v_s + sw128_offset(c, c8)) =
              make_uint4(pack_bf16(__uint_as_float(src[o]), __uint_as_float(src[o + 1])),
                         pack_bf16(__uint_as_float(src[o + 2]), __uint_as_float(src[o + 3])),
                         pack_bf16(__uint_as_float(src[o + 4]), __uint_as_float(src[o + 5])),
                         pack_bf16(__uint_as_float(src[o + 6]), __uint_as_float(src[o + 7])));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&conv_done[b]);
      // z_j[a], a = pt, once every phi thread has written its partials
      if (!(ok = mbar_wait(&z_ready[b], (n >> 1) & 1, abort_flag, status))) break;
      if (pt < D) {
        float sum = 0.f;
        #pragma unroll
        for (int r = 0; r < kRS; ++r) sum += zbuf[(b * kRS + r) * D + pt];
        h[(((size_t)bh * s.n_blocks + blk) * (D + 1) + D) * D + pt] = __float2bfloat16_rn(sum);
      }
    }
  } else {
    // ---------------------------------------------------------------- drain warps
    const int dt = tid - 320;                      // 0..127
    const int c = (warp & 3) * 32 + lane;          // my TMEM lane = row of h^T
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool ok = true;
    for (int m = 0; m < mine && ok; ++m) {
      const int b = m & 1;
      const int blk_id = blockIdx.x + m * gridDim.x;
      const int bh = blk_id / s.n_blocks, blk = blk_id % s.n_blocks;
      const int row0 = (int)(((size_t)bh * s.n_blocks + blk) * (D + 1));
      bool okl = mbar_wait(&h_full[b], (m >> 1) & 1, abort_flag, status);
      if (dt == 0 && okl) {
        bulk_wait_read_all();                      // the previous block's stores have read the tile
        mbar_arrive(out_free);
      }
      okl = okl && mbar_wait(out_free, m & 1, abort_flag, status);
      if (!(ok = __all_sync(0xFFFFFFFFu, okl))) break;
      tc_fence_after();
      #pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(lane_addr + kColH + b * 128 + cc * 32, r);
        tmem_wait_ld();
        uint8_t* box = sOut + (cc >> 1) * 16384;
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4*>(box + sw128_offset(c, (cc & 1) * 4 + i)) =
              make_uint4(pack_bf16(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                         pack_bf16(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                         pack_bf16(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                         pack_bf16(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
      }
      tc_fence_before();
      mbar_arrive(&h_free[b]);
      fence_proxy_async_smem();
      mbar_arrive(out_full);
      if (dt == 0) {
        if (!(ok = mbar_wait(out_full, m & 1, abort_flag, status))) break;
        tma_store_2d(&tmH, sOut, 0, row0);
        tma_store_2d(&tmH, sOut + 16384, 64, row0);
        bulk_commit();
      }
    }
    if (dt == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ------------------------------------------------------------------ reduce states (GEMM)
// Persistent: one CTA per SM walks the output tiles (256 query blocks x 256 state
// columns) of every head.  A tile is two M = 128 halves that share every B stage (the
// 64 K-rows x 256 columns of h), so each h slab crosses from L2 into shared memory half
// as often per output as with 128-row tiles.  A 3-stage TMA ring of 64 KB stages runs
// across tile boundaries; the two halves' accumulators fill TMEM (2 x 256 columns), so
// the epilogue hands each half back as soon as it has read it and the next tile's first
// stage starts on half 0 while half 1 drains.  Tiles are ordered M-fastest so the tiles
// sharing one slab of h run back to back (h is read from HBM about once).  Each epilogue
// warp stages its 32 rows x 64 columns per chunk in a 128B-swizzled tile and writes it
// with a TMA tensor store.
constexpr int kGemmStages = 3;
constexpr int kGemmBM = 256;
constexpr int kGemmBN = 256;
constexpr int kGemmAHalf = 128 * 128;           // 128 rows x 64 bf16
constexpr int kGemmABytes = 2 * kGemmAHalf;
constexpr int kGemmBBytes = 4 * 64 * 128;       // 4 chunks of 64 K-rows x 64 bf16
constexpr int kGemmOutBytes = 32 * 128;         // one warp's staged chunk: 32 rows x 64 bf16
constexpr int kGemmOutOff = kGemmStages * (kGemmABytes + kGemmBBytes);   // [4 warps][2 buffers]
constexpr int kGemmBarOff = kGemmOutOff + 4 * 2 * kGemmOutBytes;
constexpr int kGemmSmem = kGemmBarOff + 256 + 1024;
static_assert(kGemmSmem <= 227 * 1024, "shared memory budget");

__global__ void __launch_bounds__(192, 1)
reduce_states_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmHs, int nb, int ntot, int BH, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmStages * kGemmABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemmBarOff);
  uint64_t* full = bars;                          // [3]
  uint64_t* empty = bars + kGemmStages;           // [3]
  uint64_t* acc_full = empty + kGemmStages;       // MMA -> epilogue, one phase per tile
  uint64_t* acc_empty = acc_full + 1;             // [2] per half: epilogue -> MMA (128 arrivals)
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt_total = (nb + 63) / 64;
  const int mt = (nb + kGemmBM - 1) / kGemmBM, nt = (ntot + kGemmBN - 1) / kGemmBN;
  const int n_tiles = mt * nt * BH;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    for (int b = 0; b < 2; ++b) mbar_init(&acc_empty[b], 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      int it = 0;                                 // global k-iteration counter across tiles
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int m0 = (t % mt) * kGemmBM, n0 = ((t / mt) % nt) * kGemmBN, bh = t / (mt * nt);
        for (int kt = 0; kt < kt_total; ++kt, ++it) {
          const int s = it % kGemmStages;
          if (it >= kGemmStages && !mbar_wait(&empty[s], ((it / kGemmStages) - 1) & 1, abort_flag, status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], kGemmABytes + kGemmBBytes);
          // rows past nb (the second half of the last M tile) arrive as zero fill
          tma_load_3d(sA + s * kGemmABytes, &tmA, &full[s], kt * 64, m0, bh);
          tma_load_3d(sA + s * kGemmABytes + kGemmAHalf, &tmA, &full[s], kt * 64, m0 + 128, bh);
          for (int c = 0; c < 4; ++c)
            tma_load_3d(sB + s * kGemmBBytes + c * 8192, &tmB, &full[s], n0 + c * 64, kt * 64, bh);
        }
      }
      if (*abort_flag) {
        for (int i = (it - kGemmStages > 0 ? it - kGemmStages : 0); i < it; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[i % kGemmStages], (i / kGemmStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t id = idesc_bf16(128, kGemmBN, false, true);
      int it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++local) {
        for (int kt = 0; kt < kt_total; ++kt, ++it) {
          const int s = it % kGemmStages;
          if (!mbar_wait(&full[s], (it / kGemmStages) & 1, abort_flag, status)) { ok = false; break; }
          const uint32_t a_base = smem_u32(sA + s * kGemmABytes);
          const uint64_t b0 = desc_mnmajor(smem_u32(sB + s * kGemmBBytes), 8192);
          #pragma unroll
          for (int half = 0; half < 2; ++half) {
            // half h of the accumulator must have been read by the epilogue of tile local-1
            if (kt == 0 && local >= 1 &&
                !mbar_wait(&acc_empty[half], (local - 1) & 1, abort_flag, status)) { ok = false; break; }
            tc_fence_after();
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t a = desc_kmajor(a_base + half * kGemmAHalf + kk * 32);
              mma_bf16_ss(tmem + half * kGemmBN, a, b0 + (uint32_t)((kk * 2048) >> 4), id, (kt > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(acc_full);
      }
      if (!ok) {
        mma_commit(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else {
    // epilogue warps 0-3: TMEM lanes 32*warp.. = rows m0 + 128*half + 32*warp ..
    uint8_t* sOut = smem + kGemmOutOff + warp * 2 * kGemmOutBytes;
    int local = 0, chunk = 0;                     // chunk: this warp's store count, for the 2 staging buffers
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int m0 = (t % mt) * kGemmBM, n0 = ((t / mt) % nt) * kGemmBN, bh = t / (mt * nt);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, local & 1, abort_flag, status))) break;
      tc_fence_after();
      for (int half = 0; half < 2; ++half) {
        const int r0 = m0 + half * 128 + warp * 32;
        #pragma unroll 1
        for (int q = 0; q < kGemmBN / 64; ++q) {
          const int n = n0 + q * 64;
          if (n >= ntot) break;                    // uniform: the columns past the end have nothing to store
          uint32_t v[64];
          const uint32_t col = tmem + ((uint32_t)(warp * 32) << 16) + half * kGemmBN + q * 64;
          tmem_ld32(col, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld32(col + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          uint8_t* buf = sOut + (chunk & 1) * kGemmOutBytes;
          if (lane == 0) bulk_wait_read_1();       // the store issued from this buffer two chunks ago has read it
          __syncwarp();
          tmem_wait_ld();
          #pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint4*>(buf + sw128_offset(lane, i)) =
                make_uint4(pack_bf16(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                           pack_bf16(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                           pack_bf16(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                           pack_bf16(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past nb inside the box are clipped by the tensor map; a box wholly past
            // nb is not stored, but its (empty) group is still committed so that the
            // two-buffer wait above stays counted per chunk
            if (r0 < nb) tma_store_3d(&tmHs, buf, n, r0, bh);
            bulk_commit();
          }
          ++chunk;
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[half]);
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ------------------------------------------------------------------ linear apply
// One CTA per pair of query blocks: D_lin[t][c] = phi(q_t) . row c of [H_i'^T ; Z_i]
// (M = 128 tokens, N = d + 16, K = d), the first query block's rows written with
// TMEM lanes 64-127 masked off and the second's with lanes 0-63 masked off;
// column d holds the denominator phi(q_t) . Z_i.
template <int D>
struct ApplyLayout {
  static constexpr int kNL = D + 16;
  static constexpr int kQOff = 0;                              // phi(Q): D/64 chunks x 128 rows
  static constexpr int kHOff = kQOff + (D / 64) * 16384;       // two state tiles: D/64 chunks x kNL rows
  static constexpr int kHTile = (D / 64) * kNL * 128;
  static constexpr int kBarOff = kHOff + 2 * kHTile;
  static constexpr int kBytes = kBarOff + 64 + 1024;
};

__device__ __forceinline__ void mma_masked(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                           uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
               :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(m0), "r"(m1), "r"(m2), "r"(m3) : "memory");
}

template <int D>
__global__ void __launch_bounds__(128)
linear_apply_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmH,
                    float* __restrict__ o_lin, SeqShape s, int phi, int* status) {
  using L = ApplyLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sH = smem + L::kHOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int pair = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5;
  const bool second = 2 * pair + 1 < s.n_blocks;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const int nblk = second ? 2 : 1;
    mbar_arrive_expect_tx(&bars[0], (D / 64) * 16384 + nblk * L::kHTile);
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sQ + c * 16384, &tmQ, &bars[0], c * 64, pair * 128, bh);
      for (int b = 0; b < nblk; ++b)
        tma_load_3d(sH + b * L::kHTile + c * L::kNL * 128, &tmH, &bars[0], c * 64, 0, bh * s.n_blocks + 2 * pair + b);
    }
  }
  bool ok = cta_wait(&bars[0], 0, abort_flag, status);
  // phi(Q) in place, one row per thread; pad rows -> 0.  The softmax map takes the
  // row max in a first pass over the row and the sum of exponentials in a second.
  const int r = tid;
  const int tok = pair * 128 + r;
  const bool valid = tok < s.n_pad && token_valid(s, tok);
  if (ok) {
    float m = -INFINITY, inv = 1.f;
    if (phi == SLR_PHI_SOFTMAX) {
      #pragma unroll
      for (int gg = 0; gg < D / 8; ++gg) {
        const uint4 u = *reinterpret_cast<const uint4*>(sQ + (gg >> 3) * 16384 + sw128_offset(r, gg & 7));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(bf16_lo(w[i]), bf16_hi(w[i])));
      }
      float sum = 0.f;
      #pragma unroll
      for (int gg = 0; gg < D / 8; ++gg) {
        const uint4 u = *reinterpret_cast<const uint4*>(sQ + (gg >> 3) * 16384 + sw128_offset(r, gg & 7));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          sum += exp2f((bf16_lo(w[i]) - m) * 1.4426950408889634f) + exp2f((bf16_hi(w[i]) - m) * 1.4426950408889634f);
      }
      inv = 1.f / sum;
    }
    #pragma unroll
    for (int gg = 0; gg < D / 8; ++gg) {
      uint4* ptr = reinterpret_cast<uint4*>(sQ + (gg >> 3) * 16384 + sw128_offset(r, gg & 7));
      const uint4 u = *ptr;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o4[4];
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = bf16_lo(w[i]), b = bf16_hi(w[i]);
        if (phi == SLR_PHI_SOFTMAX) {
          a = exp2f((a - m) * 1.4426950408889634f) * inv;
          b = exp2f((b - m) * 1.4426950408889634f) * inv;
        } else {
          a = phi_elu1(a);
          b = phi_elu1(b);
        }
        o4[i] = valid ? pack_bf16(a, b) : 0u;
      }
      *ptr = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && ok) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, L::kNL, false, false);
    #pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t a = desc_kmajor(smem_u32(sQ) + (kk >> 2) * 16384 + (kk & 3) * 32);
      const uint64_t b = desc_kmajor(smem_u32(sH) + (kk >> 2) * L::kNL * 128 + (kk & 3) * 32);
      mma_masked(tmem, a, b, id, kk > 0 ? 1u : 0u, 0u, 0u, 0xFFFFFFFFu, 0xFFFFFFFFu);
    }
    if (second) {
      #pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = desc_kmajor(smem_u32(sQ) + (kk >> 2) * 16384 + (kk & 3) * 32);
        const uint64_t b = desc_kmajor(smem_u32(sH) + L::kHTile + (kk >> 2) * L::kNL * 128 + (kk & 3) * 32);
        mma_masked(tmem, a, b, id, kk > 0 ? 1u : 0u, 0xFFFFFFFFu, 0xFFFFFFFFu, 0u, 0u);
      }
    }
    mma_commit(&bars[1]);
  }
  if (ok) ok = cta_wait(&bars[1], 0, abort_flag, status);
  tc_fence_after();
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  float inv_den = 0.f;
  if (ok) {
    uint32_t dv;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(dv) : "r"(lane_addr + D));
    tmem_wait_ld();
    const float den = __uint_as_float(dv);
    inv_den = den > 0.f ? 1.f / den : 0.f;
  }
  const bool row_exists = tok < s.n_pad;
  float* out = o_lin + ((size_t)bh * s.n_pad + (row_exists ? tok : 0)) * D;
  #pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t v[32];
    if (ok) {
      tmem_ld32(lane_addr + cc * 32, v);
      tmem_wait_ld();
    }
    if (!row_exists) continue;
    float4* dst = reinterpret_cast<float4*>(out + cc * 32);
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok && valid)
        f = make_float4(__uint_as_float(v[4 * i]) * inv_den, __uint_as_float(v[4 * i + 1]) * inv_den,
                        __uint_as_float(v[4 * i + 2]) * inv_den, __uint_as_float(v[4 * i + 3]) * inv_den);
      dst[i] = f;
    }
  }
  if (!ok && tid == 0) {
    mma_commit(&bars[2]);
    const long long t0 = clock64();
    while (!mbar_try_wait(&bars[2], 0) && clock64() - t0 < kWaitBudgetCycles) {}
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 256); }
}

}  // namespace

cudaError_t launch_key_states(const void* k, const void* v, const void* w_proj, __nv_bfloat16* h, int phi, int BH,
                              int d, SeqShape s, int* status, cudaStream_t st) {
  CUtensorMap mk, mv, mw;
  const uint64_t dims[3] = {(uint64_t)d, (uint64_t)s.n_pad, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)d * 2 * s.n_pad};
  const uint32_t box[3] = {64, 64, 1};
  if (!make_tile_map(&mk, k, 3, dims, strides, box) || !make_tile_map(&mv, v, 3, dims, strides, box))
    return cudaErrorInvalidValue;
  if (w_proj) {
    const uint64_t wdims[3] = {(uint64_t)d, (uint64_t)d, 1};
    const uint64_t wstr[2] = {(uint64_t)d * 2, (uint64_t)d * 2 * d};
    const uint32_t wbox[3] = {64, (uint32_t)d, 1};
    if (!make_tile_map(&mw, w_proj, 3, wdims, wstr, wbox)) return cudaErrorInvalidValue;
  } else {
    mw = mk;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (long long)BH * s.n_blocks;
  const int grid = (int)(blocks < 2LL * sms ? blocks : 2LL * sms);
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kKsSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 128, kKsSmem, st>>>(mk, mv, mw, h, s, BH, phi, status);
    return cudaGetLastError();
  };
  if (d == 128) {
    // h viewed as rows of d values: [BH * Nb * (d + 1)][d]; the store boxes cover rows 0..d-1 of a block
    CUtensorMap mh;
    const uint64_t hdims[2] = {(uint64_t)d, (uint64_t)BH * s.n_blocks * (d + 1)};
    const uint64_t hstr[1] = {(uint64_t)d * 2};
    const uint32_t hbox[2] = {64, 128};
    if (!make_tile_map(&mh, h, 2, hdims, hstr, hbox)) return cudaErrorInvalidValue;
    const int pgrid = (int)(blocks < sms ? blocks : sms);
    auto pipe = [&](auto kern) -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, KpLayout::kBytes);
      if (e != cudaSuccess) return e;
      kern<<<pgrid, 448, KpLayout::kBytes, st>>>(mk, mv, mw, mh, h, s, BH, phi, status);
      return cudaGetLastError();
    };
    return w_proj ? pipe(key_states_pipe_kernel<true>) : pipe(key_states_pipe_kernel<false>);
  }
  return w_proj ? go(key_states_kernel<64, true>) : go(key_states_kernel<64, false>);
}

cudaError_t launch_reduce_states(const __nv_bfloat16* m01, int ld_m01, const __nv_bfloat16* h,
                                 __nv_bfloat16* Hs, int BH, int nb, int d, int* status, cudaStream_t st) {
  const int ntot = (d + 1) * d;
  CUtensorMap ma, mb, mo;
  const uint64_t adims[3] = {(uint64_t)ld_m01, (uint64_t)nb, (uint64_t)BH};
  const uint64_t astr[2] = {(uint64_t)ld_m01 * 2, (uint64_t)ld_m01 * 2 * nb};
  const uint32_t abox[3] = {64, 128, 1};
  const uint64_t bdims[3] = {(uint64_t)ntot, (uint64_t)nb, (uint64_t)BH};
  const uint64_t bstr[2] = {(uint64_t)ntot * 2, (uint64_t)ntot * 2 * nb};
  const uint32_t bbox[3] = {64, 64, 1};
  const uint32_t obox[3] = {64, 32, 1};           // Hs [BH][nb][ntot]: one warp's 32 rows x 64 columns
  if (!make_tile_map(&ma, m01, 3, adims, astr, abox) || !make_tile_map(&mb, h, 3, bdims, bstr, bbox) ||
      !make_tile_map(&mo, Hs, 3, bdims, bstr, obox))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(reduce_states_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)((nb + kGemmBM - 1) / kGemmBM) * ((ntot + kGemmBN - 1) / kGemmBN) * BH;
  const int grid = (int)(tiles < sms ? tiles : sms);
  reduce_states_kernel<<<grid, 192, kGemmSmem, st>>>(ma, mb, mo, nb, ntot, BH, status);
  return cudaGetLastError();
}

cudaError_t launch_linear_apply(const void* q, const __nv_bfloat16* Hs, float* o_lin, int phi, int BH, int d,
                                SeqShape s, int* status, cudaStream_t st) {
  CUtensorMap mq, mh;
  const uint64_t qdims[3] = {(uint64_t)d, (uint64_t)s.n_pad, (uint64_t)BH};
  const uint64_t qstr[2] = {(uint64_t)d * 2, (uint64_t)d * 2 * s.n_pad};
  const uint32_t qbox[3] = {64, 128, 1};
  const uint64_t hdims[3] = {(uint64_t)d, (uint64_t)(d + 1), (uint64_t)BH * s.n_blocks};
  const uint64_t hstr[2] = {(uint64_t)d * 2, (uint64_t)d * 2 * (d + 1)};
  const uint32_t hbox[3] = {64, (uint32_t)(d + 16), 1};
  if (!make_tile_map(&mq, q, 3, qdims, qstr, qbox) || !make_tile_map(&mh, Hs, 3, hdims, hstr, hbox))
    return cudaErrorInvalidValue;
  dim3 grid((s.n_blocks + 1) / 2, BH);
  if (d == 128) {
    cudaError_t e = cudaFuncSetAttribute(linear_apply_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, ApplyLayout<128>::kBytes);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<128><<<grid, 128, ApplyLayout<128>::kBytes, st>>>(mq, mh, o_lin, s, phi, status);
  } else {
    cudaError_t e = cudaFuncSetAttribute(linear_apply_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, ApplyLayout<64>::kBytes);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<64><<<grid, 128, ApplyLayout<64>::kBytes, st>>>(mq, mh, o_lin, s, phi, status);
  }
  return cudaGetLastError();
}

}  // namespace slr
