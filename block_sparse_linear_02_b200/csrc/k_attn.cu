// k_attn.cu -- block-sparse flash attention on tcgen05 (sm_100a).
//
// Computes, for every 64-token query block i, exact softmax attention over the
// valid keys of a set of 64-token key blocks (SLA page section 3, critical
// branch: "精确的稀疏FlashAttention"; the LVSA page's step-6 formula is the same
// normalised sum).  Two fused epilogues:
//   LINEAR  (SLA): the linear-attention branch of the same query block is added,
//           O = O_s + phi(Q_i) H_i' / (phi(Q_i) . Z_i) with H_i' = sum of
//           phi(K_j)^T V_j W_proj over its marginal blocks -- one more MMA of
//           phi(Q) against the [H_i'^T ; Z_i] rows (the last row gives the
//           denominator as an extra output column);
//   GATED   (RoPeSLR page): a far-field block of 64 pooled tokens with its own
//           softmax, combined as g*local + (1-g)*far.
//
// One CTA owns a PAIR of consecutive query blocks (128 query rows = the M of a
// tcgen05 MMA) and walks the union of their key-block sets; each list entry
// carries one flag per half, and a half that does not attend a block masks it.
// Warp roles (320 threads):
//   warp 8     TMA producer: Q once, K_j / V_j into a 3-stage ring, then the
//              linear-branch state rows;
//   warp 9     MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers; once a
//              softmax warpgroup has written its half of P_j to shared memory,
//              O_w += P_j[:, half w] V_j[half w, :];
//   warps 0-3  softmax warpgroup 0: key columns 0-31 of every block;
//   warps 4-7  softmax warpgroup 1: key columns 32-63.
// Each warpgroup runs its own online softmax (own running max and sum, own TMEM
// accumulator O_w) over its half of the keys; the epilogue merges the two
// halves exactly: O = (2^(m0-M) O_0 + 2^(m1-M) O_1) / (2^(m0-M) l_0 + 2^(m1-M) l_1).
// The softmax works in the exp2 domain with lazy rescaling (an accumulator is
// rescaled only when its running max grows by more than 2^8).
#include <cuda_runtime.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

constexpr int kStages = 3;
constexpr int kThreads = 320;
constexpr uint32_t kColO0 = 0;      // accumulator of warpgroup 0
constexpr uint32_t kColO1 = 128;    // accumulator of warpgroup 1
constexpr uint32_t kColS = 256;     // two 64-column S buffers
constexpr uint32_t kColLin = 256;   // linear branch result (reuses S after the loop)
constexpr uint32_t kColOf = 384;    // far-field accumulator

template <int D>
struct AttnLayout {
  static constexpr int kChunks = D / 64;                 // 64-column (128-byte) chunks
  static constexpr int kQChunk = 128 * 128;              // bytes of one Q chunk (128 rows)
  static constexpr int kKVChunk = 64 * 128;              // bytes of one K/V chunk (64 rows)
  static constexpr int kKVTile = kChunks * kKVChunk;
  static constexpr int kNL = D + 16;                     // rows of a linear state tile (d + z + zero pad)
  static constexpr int kHsChunk = kNL * 128;
  static constexpr int kHsTile = kChunks * kHsChunk;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kChunks * kQChunk;
  static constexpr int kVOff = kKOff + kStages * kKVTile;
  static constexpr int kPOff = kVOff + kStages * kKVTile;    // two P buffers of 128 rows x 64 keys
  static constexpr int kXOff = kPOff + 2 * 128 * 128;    // exchange area: 6 x 128 floats
  static constexpr int kBarOff = kXOff + 6 * 128 * 4;
  static constexpr int kBytes = kBarOff + 256 + 1024;    // + alignment slack
  static_assert(2 * kHsTile <= 2 * kStages * kKVTile, "linear state tiles must fit in the K/V ring");
};

struct AttnKParams {
  int n_pad, seg_len, seg_stride, n_qb, n_kb, n_pairs;
  const uint32_t* list;
  const int32_t* list_cnt;
  int list_cap, list_per_head;
  __nv_bfloat16* out;
  float* lse;
  int F, Hh, Ww, TF, TH, TW;
  float gate, scale_log2;
  int* status;
};

__device__ __forceinline__ void tile_coords(int tile, int TF, int TW, int& tf, int& th, int& tw) {
  tf = tile % TF;
  int r = tile / TF;
  tw = r % TW;
  th = r / TW;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}

// MMA with output lanes masked off (bit i of the 128-bit mask disables TMEM lane i).
__device__ __forceinline__ void mma_bf16_ss_masked(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate, const uint32_t (&mask)[4]) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
               :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate),
                  "r"(mask[0]), "r"(mask[1]), "r"(mask[2]), "r"(mask[3]) : "memory");
}

template <int D, bool TILE, bool GATED, bool LINEAR>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmX1,
            const __grid_constant__ CUtensorMap tmX2, const AttnKParams p) {
  // tmX1/tmX2: far-field K/V maps (GATED) or the linear state map (LINEAR, tmX1).
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sK = smem + L::kKOff;
  uint8_t* sV = smem + L::kVOff;
  uint8_t* sP = smem + L::kPOff;
  float* xch = reinterpret_cast<float*>(smem + L::kXOff);   // [6][128]: m0 m1 l0 l1 f0 f1
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;
  uint64_t* kv_empty = bars + 1 + 2 * kStages;
  uint64_t* s_full = bars + 1 + 3 * kStages;     // [2]  per S buffer
  uint64_t* p_full = s_full + 2;                 // [4]  [warpgroup * 2 + P buffer]
  uint64_t* o_bar = p_full + 4;                  // [4]  [warpgroup * 2 + P buffer]
  uint64_t* loop_done = o_bar + 4;
  uint64_t* hs_full = loop_done + 1;
  uint64_t* phiq_ready = hs_full + 1;
  uint64_t* lin_done = phiq_ready + 1;
  uint64_t* far_x = lin_done + 1;               // far-field max exchange between the warpgroups
  uint64_t* drain = far_x + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  constexpr uint32_t kTmemCols = 512;

  const uint32_t* list = nullptr;
  int n_local = p.n_kb;
  if (p.list) {
    size_t off = (p.list_per_head ? (size_t)bh * p.n_pairs : 0) + pair;
    list = p.list + off * p.list_cap;
    n_local = p.list_cnt[off];
  }
  const int total = n_local + (GATED ? 1 : 0);
  const bool second_exists = 2 * pair + 1 < p.n_qb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&k_full[s], 1); mbar_init(&v_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    for (int i = 0; i < 4; ++i) { mbar_init(&p_full[i], 128); mbar_init(&o_bar[i], 1); }
    mbar_init(loop_done, 1);
    mbar_init(hs_full, 1);
    mbar_init(phiq_ready, 256);
    mbar_init(lin_done, 1);
    mbar_init(far_x, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, L::kChunks * L::kQChunk);
      if (TILE) {
        for (int half = 0; half < 2; ++half) {
          int tf, th, tw;
          tile_coords(2 * pair + half, p.TF, p.TW, tf, th, tw);
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_5d(sQ + c * L::kQChunk + half * L::kKVChunk, &tmQ, q_full, c * 64, tw * 4, th * 4, tf * 4, bh);
        }
      } else {
        for (int c = 0; c < L::kChunks; ++c) tma_load_3d(sQ + c * L::kQChunk, &tmQ, q_full, c * 64, pair * 128, bh);
      }
      int j = 0;
      for (; j < total; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(&kv_empty[s], ((j / kStages) - 1) & 1, abort_flag, p.status)) break;
        const bool far = GATED && j == n_local;
        const int kb = far ? 0 : (list ? (int)(list[j] & 0x3FFFFFFFu) : j);
        uint8_t* dK = sK + s * L::kKVTile;
        uint8_t* dV = sV + s * L::kKVTile;
        mbar_arrive_expect_tx(&k_full[s], L::kKVTile);
        mbar_arrive_expect_tx(&v_full[s], L::kKVTile);
        if (far) {
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dK + c * L::kKVChunk, &tmX1, &k_full[s], c * 64, 0, bh);
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dV + c * L::kKVChunk, &tmX2, &v_full[s], c * 64, 0, bh);
        } else if (TILE) {
          int tf, th, tw;
          tile_coords(kb, p.TF, p.TW, tf, th, tw);
          for (int c = 0; c < L::kChunks; ++c) tma_load_5d(dK + c * L::kKVChunk, &tmK, &k_full[s], c * 64, tw * 4, th * 4, tf * 4, bh);
          for (int c = 0; c < L::kChunks; ++c) tma_load_5d(dV + c * L::kKVChunk, &tmV, &v_full[s], c * 64, tw * 4, th * 4, tf * 4, bh);
        } else {
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dK + c * L::kKVChunk, &tmK, &k_full[s], c * 64, kb * 64, bh);
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dV + c * L::kKVChunk, &tmV, &v_full[s], c * 64, kb * 64, bh);
        }
      }
      if (LINEAR && j == total && mbar_wait(loop_done, 0, abort_flag, p.status)) {
        // the K/V ring is free: bring in the [H'^T ; Z] rows of both query blocks
        const int nblk = second_exists ? 2 : 1;
        mbar_arrive_expect_tx(hs_full, nblk * L::kHsTile);
        for (int b = 0; b < nblk; ++b)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_3d(sK + b * L::kHsTile + c * L::kHsChunk, &tmX1, hs_full, c * 64, 0,
                        bh * p.n_qb + 2 * pair + b);
      }
      if (*abort_flag) {
        for (int i = (j - kStages > 0 ? j - kStages : 0); i < j; ++i) {
          const int s = i % kStages;
          const long long t0 = clock64();
          while (!mbar_try_wait(&k_full[s], (i / kStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
          while (!mbar_try_wait(&v_full[s], (i / kStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && total > 0) {
      constexpr uint32_t idS = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV), p_addr = smem_u32(sP);
      auto issue_qk = [&](int stage, int sbuf) {
        #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, sub = kk & 3;
          uint64_t a = desc_kmajor(q_addr + c * L::kQChunk + sub * 32);
          uint64_t b = desc_kmajor(k_addr + stage * L::kKVTile + c * L::kKVChunk + sub * 32);
          mma_bf16_ss(tmem + kColS + sbuf * 64, a, b, idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int stage, int pbuf, uint32_t col, int kk0, int kk1, bool acc) {
        for (int kk = kk0; kk < kk1; ++kk) {
          uint64_t a = desc_kmajor(p_addr + pbuf * 16384 + kk * 32);
          uint64_t b = desc_mnmajor(v_addr + stage * L::kKVTile + kk * 2048, L::kKVChunk);
          mma_bf16_ss(tmem + col, a, b, idO, (acc || kk > kk0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status) && mbar_wait(&k_full[0], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&s_full[0]);
        for (int j = 0; j < total && ok; ++j) {
          if (j + 1 < total) {
            const int s1 = (j + 1) % kStages;
            if (!mbar_wait(&k_full[s1], ((j + 1) / kStages) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_qk(s1, (j + 1) & 1);
            mma_commit(&s_full[(j + 1) & 1]);
          }
          const int s = j % kStages;
          if (!mbar_wait(&v_full[s], (j / kStages) & 1, abort_flag, p.status)) { ok = false; break; }
          const bool far = GATED && j == n_local;
          const int pb = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (far) {
            if (!mbar_wait(&p_full[pb], ph, abort_flag, p.status) ||
                !mbar_wait(&p_full[2 + pb], ph, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(s, pb, kColOf, 0, 4, false);
            mma_commit(&o_bar[pb]);
            mma_commit(&o_bar[2 + pb]);
          } else {
            if (!mbar_wait(&p_full[pb], ph, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(s, pb, kColO0, 0, 2, j > 0);
            mma_commit(&o_bar[pb]);
            if (!mbar_wait(&p_full[2 + pb], ph, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(s, pb, kColO1, 2, 4, j > 0);
            mma_commit(&o_bar[2 + pb]);
          }
          mma_commit(&kv_empty[s]);
        }
        if (ok) mma_commit(loop_done);
        if (ok && LINEAR) {
          ok = mbar_wait(hs_full, 0, abort_flag, p.status) && mbar_wait(phiq_ready, 0, abort_flag, p.status);
          if (ok) {
            tc_fence_after();
            constexpr uint32_t idL = idesc_bf16(128, L::kNL, false, false);
            const uint32_t lo_only[4] = {0u, 0u, 0xFFFFFFFFu, 0xFFFFFFFFu};   // write lanes 0-63
            const uint32_t hi_only[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0u, 0u};   // write lanes 64-127
            #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int c = kk >> 2, sub = kk & 3;
              const uint64_t a = desc_kmajor(q_addr + c * L::kQChunk + sub * 32);
              const uint64_t b = desc_kmajor(k_addr + c * L::kHsChunk + sub * 32);
              mma_bf16_ss_masked(tmem + kColLin, a, b, idL, kk > 0 ? 1u : 0u, lo_only);
            }
            if (second_exists) {
              #pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const int c = kk >> 2, sub = kk & 3;
                const uint64_t a = desc_kmajor(q_addr + c * L::kQChunk + sub * 32);
                const uint64_t b = desc_kmajor(k_addr + L::kHsTile + c * L::kHsChunk + sub * 32);
                mma_bf16_ss_masked(tmem + kColLin, a, b, idL, kk > 0 ? 1u : 0u, hi_only);
              }
            }
            mma_commit(lin_done);
          }
        }
      }
      if (!ok) {
        mma_commit(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int wg = warp >> 2;                  // 0: key columns 0-31, 1: columns 32-63
    const int r = threadIdx.x & 127;           // query row of the pair = TMEM lane
    const int half = r >> 6;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t my_o = wg ? kColO1 : kColO0;
    const float sl = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f, m_far = -INFINITY, l_far = 0.f;
    const SeqShape seq{p.n_pad, p.seg_len, p.seg_stride, p.n_kb};
    bool ok = true;
    for (int j = 0; j < total; ++j) {
      const bool far = GATED && j == n_local;
      const int sb = j & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag, p.status))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(lane_addr + kColS + sb * 64 + wg * 32, sr);
      int nvalid = 64;
      bool attend = true;
      if (!far) {
        const uint32_t e = list ? list[j] : ((uint32_t)j | 0xC0000000u);
        attend = (e >> (30 + half)) & 1u;
        if (!TILE) nvalid = block_valid_count(seq, (int)(e & 0x3FFFFFFFu));
      }
      const int lo = wg * 32;
      const bool none = !attend || nvalid <= lo;
      const bool full = attend && nvalid >= lo + 32;
      tmem_wait_ld();
      float mx = -INFINITY;
      if (full) {
        float t[11];
        #pragma unroll
        for (int i = 0; i < 10; ++i)
          t[i] = max3(__uint_as_float(sr[3 * i]), __uint_as_float(sr[3 * i + 1]), __uint_as_float(sr[3 * i + 2]));
        t[10] = fmaxf(__uint_as_float(sr[30]), __uint_as_float(sr[31]));
        const float u0 = max3(t[0], t[1], t[2]), u1 = max3(t[3], t[4], t[5]), u2 = max3(t[6], t[7], t[8]);
        mx = max3(max3(u0, u1, u2), t[9], t[10]);
      } else if (!none) {
        #pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (lo + c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
          mx = fmaxf(mx, __uint_as_float(sr[c]));
        }
      }
      float m_new;
      if (far) {
        // both warpgroups share the far block's max so that its P is one consistent row
        xch[(4 + wg) * 128 + r] = none ? -INFINITY : mx;
        mbar_arrive(far_x);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(far_x, 0, abort_flag, p.status))) { ok = false; break; }
        const float other = xch[(5 - wg) * 128 + r];
        m_new = fmaxf(none ? -INFINITY : mx, other) * sl;
        m_far = m_new;
      } else {
        m_new = fmaxf(m_run, mx * sl);
      }
      float factor = 1.f;
      bool need = false;
      if (!far) {
        need = m_new > m_run + 8.f;
        if (need) {
          factor = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
          l_run *= factor;
          m_run = m_new;
        }
      }
      const float mcur = far ? m_far : m_run;
      const float mu = (mcur == -INFINITY) ? 0.f : mcur;
      uint32_t packed[16];
      float rowsum = 0.f;
      if (none) {
        #pragma unroll
        for (int c = 0; c < 16; ++c) packed[c] = 0u;
      } else {
        float acc0 = 0.f, acc1 = 0.f;
        #pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(sr[c]), sl, -mu));
          const float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), sl, -mu));
          acc0 += p0;
          acc1 += p1;
          packed[c >> 1] = pack_bf16(p0, p1);
        }
        rowsum = acc0 + acc1;
      }
      if (far) l_far += rowsum; else l_run += rowsum;
      // P buffer j&1 (my half) is free once P_{j-2} V_{j-2} has completed; my accumulator
      // may be rescaled once P_{j-1} V_{j-1} has completed
      const int pb = j & 1;
      if (j >= 2) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&o_bar[wg * 2 + pb], ((j - 2) >> 1) & 1, abort_flag, p.status))) { ok = false; break; }
      }
      const bool rescale = !far && j > 0 && __any_sync(0xFFFFFFFFu, need);
      if (rescale) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&o_bar[wg * 2 + (pb ^ 1)], ((j - 1) >> 1) & 1, abort_flag, p.status))) { ok = false; break; }
      }
      tc_fence_after();
      if (rescale) {
        #pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_addr + my_o + cc * 32, o);
          tmem_wait_ld();
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(lane_addr + my_o + cc * 32, o);
        }
        tmem_wait_st();
      }
      #pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint4 val = make_uint4(packed[4 * c8], packed[4 * c8 + 1], packed[4 * c8 + 2], packed[4 * c8 + 3]);
        *reinterpret_cast<uint4*>(sP + pb * 16384 + sw128_offset(r, 4 * wg + c8)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[wg * 2 + pb]);
    }
    if (ok && total > 0)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&o_bar[wg * 2 + ((total - 1) & 1)], ((total - 1) >> 1) & 1, abort_flag, p.status));
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();

    // ---- token of this row
    int tok;
    bool row_exists;
    if (TILE) {
      const int tile = 2 * pair + half;
      row_exists = tile < p.n_qb;
      int tf, th, tw;
      tile_coords(tile, p.TF, p.TW, tf, th, tw);
      const int rr = r & 63;
      tok = ((tf * 4 + (rr >> 4)) * p.Hh + th * 4 + ((rr >> 2) & 3)) * p.Ww + tw * 4 + (rr & 3);
    } else {
      tok = pair * 128 + r;
      row_exists = tok < p.n_pad;
    }
    const bool valid = row_exists && (TILE || token_valid(seq, tok));

    bool lin_ok = false;
    if (LINEAR) {
      // phi(Q) in place (the last QK MMA has completed); pad rows -> 0
      if (ok) {
        constexpr int kGroups = D / 16;                  // 16-byte groups of my row handled by my warpgroup
        #pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          const int gg = wg * kGroups + g;               // 0 .. D/8-1
          uint4* ptr = reinterpret_cast<uint4*>(sQ + (gg >> 3) * L::kQChunk + sw128_offset(r, gg & 7));
          const uint4 u = *ptr;
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          uint32_t o4[4];
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            o4[i] = valid ? pack_bf16(phi_elu1(bf16_lo(w[i])), phi_elu1(bf16_hi(w[i]))) : 0u;
          *ptr = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(phiq_ready);
      if (ok) lin_ok = __all_sync(0xFFFFFFFFu, mbar_wait(lin_done, 0, abort_flag, p.status));
      tc_fence_after();
    }

    // ---- merge the two halves
    xch[wg * 128 + r] = m_run;
    xch[(2 + wg) * 128 + r] = l_run;
    if (GATED) xch[(4 + wg) * 128 + r] = l_far;
    softmax_bar();
    const float m0 = xch[r], m1 = xch[128 + r], l0 = xch[256 + r], l1 = xch[384 + r];
    const float M = fmaxf(m0, m1);
    const float a0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
    const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
    const float Lsum = a0 * l0 + a1 * l1;
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const float c0 = a0 * inv, c1 = a1 * inv;
    float inv_far = 0.f;
    if (GATED) {
      const float lf = xch[512 + r] + xch[640 + r];
      inv_far = lf > 0.f ? 1.f / lf : 0.f;
    }
    float inv_den = 0.f;
    if (LINEAR && lin_ok) {
      uint32_t dv;
      tmem_ld1(lane_addr + kColLin + D, dv);
      tmem_wait_ld();
      const float den = __uint_as_float(dv);
      inv_den = den > 0.f ? 1.f / den : 0.f;
    }
    const bool have_o = ok && n_local > 0;         // CTA-uniform
    const size_t row_off = ((size_t)bh * p.n_pad + (row_exists ? tok : 0)) * D;
    #pragma unroll 1
    for (int cc = wg * (D / 64); cc < (wg + 1) * (D / 64); ++cc) {
      float v[32];
      if (have_o) {
        uint32_t o0[32], o1[32];
        tmem_ld32(lane_addr + kColO0 + cc * 32, o0);
        tmem_ld32(lane_addr + kColO1 + cc * 32, o1);
        tmem_wait_ld();
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = c0 * __uint_as_float(o0[i]) + c1 * __uint_as_float(o1[i]);
      } else {
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (GATED && ok) {
        uint32_t of[32];
        tmem_ld32(lane_addr + kColOf + cc * 32, of);
        tmem_wait_ld();
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = p.gate * v[i] + (1.f - p.gate) * (__uint_as_float(of[i]) * inv_far);
      }
      if (LINEAR && lin_ok) {
        uint32_t ol[32];
        tmem_ld32(lane_addr + kColLin + cc * 32, ol);
        tmem_wait_ld();
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += __uint_as_float(ol[i]) * inv_den;
      }
      if (!row_exists) continue;
      uint4* dst = reinterpret_cast<uint4*>(p.out + row_off + cc * 32);
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w4 = make_uint4(0, 0, 0, 0);
        if (valid)
          w4 = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
        dst[i] = w4;
      }
    }
    if (p.lse && row_exists && wg == 0) {
      float val = 0.f;
      if (valid) val = (Lsum > 0.f) ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
      p.lse[(size_t)bh * p.n_pad + tok] = val;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool TILE, bool GATED, bool LINEAR>
cudaError_t launch_variant(const AttnArgs& a, const CUtensorMap* maps, const AttnKParams& kp, cudaStream_t st) {
  using L = AttnLayout<D>;
  auto kern = attn_kernel<D, TILE, GATED, LINEAR>;
  static unsigned long long attr_set = 0;        // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  dim3 grid(a.n_pairs, a.BH);
  kern<<<grid, kThreads, L::kBytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], kp);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap* maps, const AttnKParams& kp, cudaStream_t st) {
  if (a.tile3d) return launch_variant<D, true, true, false>(a, maps, kp, st);
  if (a.Hs) return launch_variant<D, false, false, true>(a, maps, kp, st);
  return launch_variant<D, false, false, false>(a, maps, kp, st);
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  const int D = a.d;
  if (a.tile3d && !a.gated) return cudaErrorInvalidValue;
  CUtensorMap maps[5];
  const uint64_t rowb = (uint64_t)D * 2;
  if (a.tile3d) {
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)a.Ww, (uint64_t)a.Hh, (uint64_t)a.F, (uint64_t)a.BH};
    const uint64_t strides[4] = {rowb, rowb * a.Ww, rowb * a.Ww * a.Hh, rowb * a.Ww * a.Hh * a.F};
    const uint32_t box[5] = {64, 4, 4, 4, 1};
    if (!make_tile_map(&maps[0], a.q, 5, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[1], a.k, 5, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[2], a.v, 5, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.s.n_pad, (uint64_t)a.BH};
    const uint64_t strides[2] = {rowb, rowb * a.s.n_pad};
    const uint32_t boxq[3] = {64, 128, 1};
    const uint32_t boxkv[3] = {64, 64, 1};
    if (!make_tile_map(&maps[0], a.q, 3, dims, strides, boxq)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[1], a.k, 3, dims, strides, boxkv)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[2], a.v, 3, dims, strides, boxkv)) return cudaErrorInvalidValue;
  }
  maps[3] = maps[1];
  maps[4] = maps[2];
  if (a.gated) {
    const uint64_t dims[3] = {(uint64_t)D, 64, (uint64_t)a.BH};
    const uint64_t strides[2] = {rowb, rowb * 64};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tile_map(&maps[3], a.kf, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[4], a.vf, 3, dims, strides, box)) return cudaErrorInvalidValue;
  } else if (a.Hs) {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(D + 1), (uint64_t)a.BH * a.n_qb};
    const uint64_t strides[2] = {rowb, rowb * (D + 1)};
    const uint32_t box[3] = {64, (uint32_t)(D + 16), 1};
    if (!make_tile_map(&maps[3], a.Hs, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  AttnKParams kp;
  kp.n_pad = a.s.n_pad; kp.seg_len = a.s.seg_len; kp.seg_stride = a.s.seg_stride;
  kp.n_qb = a.n_qb; kp.n_kb = a.n_kb; kp.n_pairs = a.n_pairs;
  kp.list = a.list; kp.list_cnt = a.list_cnt; kp.list_cap = a.list_cap; kp.list_per_head = a.list_per_head;
  kp.out = reinterpret_cast<__nv_bfloat16*>(a.out); kp.lse = a.lse;
  kp.F = a.F; kp.Hh = a.Hh; kp.Ww = a.Ww;
  kp.TF = a.tile3d ? a.F / 4 : 1; kp.TH = a.tile3d ? a.Hh / 4 : 1; kp.TW = a.tile3d ? a.Ww / 4 : 1;
  kp.gate = a.gate;
  kp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  kp.status = a.status;
  return D == 128 ? launch_d<128>(a, maps, kp, st) : launch_d<64>(a, maps, kp, st);
}

}  // namespace slr
