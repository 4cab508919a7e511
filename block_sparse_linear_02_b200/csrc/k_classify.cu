// k_classify.cu -- SLA's compressed scores, percentile classification and the
// critical pair lists.
//
// SLA page section 3: the pooled Q and K give a compressed attention-weight
// matrix P_c = softmax(pool(Q) pool(K)^T / sqrt(d)); within each query-block row
// the top 5 % positions are labelled critical (1), the bottom 10 % negligible
// (-1), the rest marginal (0).  Softmax is strictly increasing along a row, so
// the labels are taken on the logits qbar_i . kbar_j; ties rank the lower
// key-block index first.
//
// logits_kernel: one CTA per 128 x 128 tile of one head's logit matrix on the
//   tensor cores.  The pooling kernel writes each mean as a bf16 pair hi + lo,
//   query rows as [qh | qh | ql] and key rows as [kh | kl | kh], so one bf16
//   GEMM over K = 3d with fp32 accumulation gives qh.kh + qh.kl + ql.kh: the
//   logit up to the ql.kl term, about 2^-16 of it.  The tile is stored as
//   order-preserving 32-bit keys (pad columns 0).
// classify_kernel: one warp per pair of query blocks.  For both rows, the kc-th
//   largest and the kn-th smallest key by bisection (one comparison per key and
//   one warp sum per bit); then one pass in index order applies the thresholds
//   with index tie-breaking and writes what the caller asked for: the mask row,
//   the ascending critical list, the marginal indicator m01 (bf16 1/0, the
//   operand of the tensor-core contraction), P_c in fp32, and the pair's union
//   list for the attention kernel.
// Against an exact evaluation the logits' error moves P_c by ~1e-8, so a label
// can differ only for a pair whose score is that close to its row's threshold.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

// Order-preserving map of an fp32 value onto uint32 (larger value -> larger key);
// -0 is folded onto +0 so that equal values give equal keys.  A finite value
// never maps to 0, which marks padding.
__device__ __forceinline__ uint32_t okey(float x) {
  if (x == 0.f) x = 0.f;
  const uint32_t b = __float_as_uint(x);
  return (b >> 31) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float okey_value(uint32_t k) {
  return __uint_as_float((k >> 31) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ int warp_sum(int v) { return (int)__reduce_add_sync(0xFFFFFFFFu, (unsigned)v); }

// ------------------------------------------------------------------ logits GEMM
// One 128x128 logit tile per CTA, K = 3d streamed through a 3-stage ring of (A, B)
// 64-column chunks, so that two CTAs fit on an SM and the tiles of a head run in one
// wave.  Roles: thread 0 loads, thread 32 issues the MMAs; then every warp turns its
// 32 rows into keys, stages them 128B-swizzled in the (then idle) ring and writes
// them with TMA tensor stores.
template <int D>
struct LgLayout {
  static constexpr int kChunks = 3 * D / 64;          // K = 3d in chunks of 64
  static constexpr int kTile = 128 * 128;             // 128 rows x 64 bf16
  static constexpr int kStages = 3;
  static constexpr int kStage = 2 * kTile;            // A chunk, then B chunk
  static constexpr int kOutChunk = 32 * 128;          // one warp's 32 rows x 32 keys
  static constexpr int kBarOff = kStages * kStage;
  static constexpr int kBytes = kBarOff + 256 + 1024; // + alignment slack
  static_assert(16 * kOutChunk <= kStages * kStage, "key staging reuses the ring");
};

template <int D>
__global__ void __launch_bounds__(128, 2)
logits_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmKeys, int nb, int nbp, int* status) {
  using L = LgLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);   // [kStages]
  uint64_t* empty = full + L::kStages;                              // [kStages]
  uint64_t* done = empty + L::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * 128, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) {
    // ---- loads
    int issued = 0;
    for (int c = 0; c < L::kChunks; ++c) {
      const int s = c % L::kStages;
      if (c >= L::kStages && !mbar_wait(&empty[s], ((c / L::kStages) - 1) & 1, abort_flag, status)) break;
      mbar_arrive_expect_tx(&full[s], L::kStage);
      tma_load_3d(smem + s * L::kStage, &tmA, &full[s], c * 64, m0, bh);
      tma_load_3d(smem + s * L::kStage + L::kTile, &tmB, &full[s], c * 64, n0, bh);
      ++issued;
    }
    if (*abort_flag) {
      // let the loads in flight land before the shared memory is released
      for (int c = (issued > L::kStages ? issued - L::kStages : 0); c < issued; ++c) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&full[c % L::kStages], (c / L::kStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (threadIdx.x == 32) {
    // ---- MMAs
    constexpr uint32_t id = idesc_bf16(128, 128, false, false);
    for (int c = 0; c < L::kChunks; ++c) {
      const int s = c % L::kStages;
      if (!mbar_wait(&full[s], (c / L::kStages) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t base = smem_u32(smem + s * L::kStage);
      #pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem, desc_kmajor(base + kk * 32), desc_kmajor(base + L::kTile + kk * 32), id,
                    (c > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&empty[s]);
    }
    mma_commit(done);   // also when aborting: the MMAs already issued complete before the CTA exits
  }
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(done, 0, abort_flag, status)) && !*abort_flag;
  tc_fence_after();
  __syncthreads();                          // every role is past the ring before it is reused
  if (ok) {                                 // warp-uniform: the TMEM loads are warp-collective
    const int row0 = m0 + warp * 32;
    #pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + cc * 32, v);
      tmem_wait_ld();
      #pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = n0 + cc * 32 + i < nb ? okey(__uint_as_float(v[i])) : 0u;
      uint8_t* buf = smem + (warp * 4 + cc) * L::kOutChunk;
      #pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint4*>(buf + sw128_offset(lane, i)) = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      // the keys moved as bf16 pairs: 32 keys = 64 elements; rows past nb are clipped
      if (lane == 0 && row0 < nb) {
        tma_store_3d(&tmKeys, buf, 2 * (n0 + cc * 32), row0, bh);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 128); }
}

// ------------------------------------------------------------------ classification
struct ClsArgs {
  const uint32_t* keys;    // [BH][nb][nbp] order keys of the logits, pads 0
  int nb, nbp, kc, kn, n_pairs;
  float inv_sqrt_d;
  int8_t* mask;
  bool mask_vec;           // rows of the mask can take 4-byte stores (nb % 4 == 0, 4-byte aligned base)
  int32_t* crit_idx;
  int32_t* crit_cnt;
  __nv_bfloat16* m01;
  int ld_m01;
  float* scores;
  uint32_t* list;
  int32_t* list_cnt;
  int list_cap;
  SeqShape s;
  int* status;
};

constexpr int kClsWarps = 4;
constexpr int kPrefixBits = 12;      // thresholds are first located to the top 12 key bits
constexpr int kMaxCand = 32;         // candidates resolved exactly by ranking

__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// One warp per pair of query blocks.  Each row's keys sit in shared memory; lane l
// owns keys 128 g + 4 l .. +3 of every 128-key group g (one 16-byte load).
//   1. Bisection over the top kPrefixBits key bits: Tc = prefix of the kc-th
//      largest key, Tn = prefix of the kn-th smallest.
//   2. The keys sharing the threshold prefix (a handful, since the prefix fixes
//      sign, exponent and 3 mantissa bits) are collected and ranked exactly; if
//      more than kMaxCand share a prefix the bisection continues over the
//      remaining bits instead.
//   3. One pass in index order writes the labels and outputs; ties at a threshold
//      go to the lower index (critical) or leave the higher index marginal
//      (negligible), via warp prefix counts of the tied keys.
__global__ void __launch_bounds__(kClsWarps * 32, 6)
classify_kernel(const ClsArgs a) {
  extern __shared__ __align__(16) uint32_t skeys[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, pair = blockIdx.x * kClsWarps + warp;
  const int nb = a.nb, nbp = a.nbp, ng = nbp / 128;
  const int qb0 = 2 * pair;
  if (qb0 >= nb) return;
  const int nrows = qb0 + 1 < nb ? 2 : 1;
  uint32_t* rowk[2] = {skeys + (size_t)(2 * warp) * nbp, skeys + (size_t)(2 * warp + 1) * nbp};
  uint32_t* cand = skeys + (size_t)kClsWarps * 2 * nbp + warp * (4 * kMaxCand);   // [4][kMaxCand]
  int ccount[4] = {0, 0, 0, 0};
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < nrows; ++r) {
    const uint4* src = reinterpret_cast<const uint4*>(a.keys + ((size_t)bh * nb + qb0 + r) * nbp);
    for (int e = lane; e < nbp / 4; e += 32) reinterpret_cast<uint4*>(rowk[r])[e] = src[e];
  }
  __syncwarp();
  const int npad = nbp - nb;

  // ---- 1. thresholds to kPrefixBits bits (pads are key 0: never >= a candidate
  // top threshold, always <= a candidate bottom one)
  uint32_t Tc[2] = {0u, 0u}, Tn[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
  auto bisect = [&](int hi, int lo) {
    for (int bit = hi; bit >= lo; --bit) {
      #pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r >= nrows) break;                    // warp-uniform
        const uint32_t cc = Tc[r] | (1u << bit), cn = Tn[r] & ~(1u << bit);
        int nc = 0, nn = 0;
        for (int g = 0; g < ng; ++g) {
          const uint4 k4 = *reinterpret_cast<const uint4*>(rowk[r] + g * 128 + lane * 4);
          nc += (k4.x >= cc) + (k4.y >= cc) + (k4.z >= cc) + (k4.w >= cc);
          nn += (k4.x <= cn) + (k4.y <= cn) + (k4.z <= cn) + (k4.w <= cn);
        }
        if (warp_sum(nc) >= a.kc) Tc[r] = cc;
        if (warp_sum(nn) - npad >= a.kn) Tn[r] = cn;
      }
    }
  };
  bisect(31, 32 - kPrefixBits);

  // ---- 2. exact thresholds: collect the keys that share each threshold prefix
  constexpr int kSh = 32 - kPrefixBits;
  int gt_c[2] = {0, 0}, lt_n[2] = {0, 0}, eq_n[2] = {0, 0};
  #pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (r >= nrows) break;
    const uint32_t pc = Tc[r] >> kSh, pn = Tn[r] >> kSh;
    int gt = 0, lt = 0;
    for (int g = 0; g < ng; ++g) {
      const uint4 k4 = *reinterpret_cast<const uint4*>(rowk[r] + g * 128 + lane * 4);
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t pk = kk[i] >> kSh;
        gt += pk > pc;
        lt += kk[i] != 0u && pk < pn;
        // keys sharing a threshold prefix, appended in ballot order (their order is irrelevant)
        const unsigned mc = __ballot_sync(0xFFFFFFFFu, pk == pc);
        if (mc) {
          const int at = ccount[2 * r] + __popc(mc & lt_mask);
          if (pk == pc && at < kMaxCand) cand[(2 * r) * kMaxCand + at] = kk[i];
          ccount[2 * r] += __popc(mc);
        }
        const unsigned mn = __ballot_sync(0xFFFFFFFFu, kk[i] != 0u && pk == pn);
        if (mn) {
          const int at = ccount[2 * r + 1] + __popc(mn & lt_mask);
          if (kk[i] != 0u && pk == pn && at < kMaxCand) cand[(2 * r + 1) * kMaxCand + at] = kk[i];
          ccount[2 * r + 1] += __popc(mn);
        }
      }
    }
    gt_c[r] = warp_sum(gt);
    lt_n[r] = warp_sum(lt);
  }
  __syncwarp();
  bool fits = true;
  for (int r = 0; r < nrows; ++r) fits = fits && ccount[2 * r] <= kMaxCand && (a.kn == 0 || ccount[2 * r + 1] <= kMaxCand);
  if (fits) {
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r >= nrows) break;
      // top: the (kc - gt)-th largest candidate; lane l ranks candidate l
      {
        const int n = ccount[2 * r], need = a.kc - gt_c[r];
        const uint32_t c = lane < n ? cand[(2 * r) * kMaxCand + lane] : 0u;
        int above = 0, atleast = 0;
        for (int m = 0; m < n; ++m) {
          const uint32_t o = cand[(2 * r) * kMaxCand + m];
          above += o > c;
          atleast += o >= c;
        }
        const bool is_t = lane < n && above < need && need <= atleast;
        const unsigned bt = __ballot_sync(0xFFFFFFFFu, is_t);
        const int src = __ffs(bt) - 1;
        Tc[r] = __shfl_sync(0xFFFFFFFFu, c, src);
        gt_c[r] += __shfl_sync(0xFFFFFFFFu, above, src);
      }
      if (a.kn > 0) {
        const int n = ccount[2 * r + 1], need = a.kn - lt_n[r];
        const uint32_t c = lane < n ? cand[(2 * r + 1) * kMaxCand + lane] : 0xFFFFFFFFu;
        int below = 0, atmost = 0;
        for (int m = 0; m < n; ++m) {
          const uint32_t o = cand[(2 * r + 1) * kMaxCand + m];
          below += o < c;
          atmost += o <= c;
        }
        const bool is_t = lane < n && below < need && need <= atmost;
        const unsigned bt = __ballot_sync(0xFFFFFFFFu, is_t);
        const int src = __ffs(bt) - 1;
        Tn[r] = __shfl_sync(0xFFFFFFFFu, c, src);
        lt_n[r] += __shfl_sync(0xFFFFFFFFu, below, src);
        eq_n[r] = __shfl_sync(0xFFFFFFFFu, atmost - below, src);
      }
    }
  } else {
    // many keys share a prefix (e.g. tied rows): finish the bisection and count
    bisect(31 - kPrefixBits, 0);
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r >= nrows) break;
      int gt = 0, lt = 0, eq = 0;
      for (int g = 0; g < ng; ++g) {
        const uint4 k4 = *reinterpret_cast<const uint4*>(rowk[r] + g * 128 + lane * 4);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          gt += kk[i] > Tc[r];
          lt += kk[i] != 0u && kk[i] < Tn[r];
          eq += kk[i] == Tn[r];
        }
      }
      gt_c[r] = warp_sum(gt);
      lt_n[r] = warp_sum(lt);
      eq_n[r] = warp_sum(eq);
    }
  }

  // ---- P_c normaliser (only when scores are requested)
  float row_max[2] = {0.f, 0.f}, row_sum[2] = {1.f, 1.f};
  if (a.scores) {
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r >= nrows) break;
      uint32_t kmax = 0u;
      for (int j = lane; j < nb; j += 32) kmax = rowk[r][j] > kmax ? rowk[r][j] : kmax;
      row_max[r] = okey_value(__reduce_max_sync(0xFFFFFFFFu, kmax));
      float sum = 0.f;
      for (int j = lane; j < nb; j += 32) sum += expf((okey_value(rowk[r][j]) - row_max[r]) * a.inv_sqrt_d);
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      row_sum[r] = sum;
    }
  }

  // ---- 3. labels in index order and the outputs
  int seen_c[2] = {0, 0}, seen_n[2] = {0, 0}, written[2] = {0, 0}, listed = 0;
  (void)lt_mask;
  uint32_t* lst = a.list ? a.list + ((size_t)bh * a.n_pairs + pair) * a.list_cap : nullptr;
  for (int g = 0; g < ng; ++g) {
    const int j0 = g * 128 + lane * 4;           // my 4 keys: j0 .. j0+3
    uint32_t crit_bits[2] = {0u, 0u};
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r >= nrows) break;
      const uint4 k4 = *reinterpret_cast<const uint4*>(rowk[r] + g * 128 + lane * 4);
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
      uint32_t gtb = 0, eqcb = 0, ltb = 0, eqnb = 0;
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool in = j0 + i < nb;
        gtb |= (uint32_t)(in && kk[i] > Tc[r]) << i;
        eqcb |= (uint32_t)(in && kk[i] == Tc[r]) << i;
        ltb |= (uint32_t)(in && kk[i] < Tn[r]) << i;
        eqnb |= (uint32_t)(in && kk[i] == Tn[r]) << i;
      }
      // critical: all above Tc, plus the first (kc - gt_c) keys equal to Tc in index order
      uint32_t cb = gtb;
      if (__any_sync(0xFFFFFFFFu, eqcb != 0u)) {
        const int ne = __popc(eqcb);
        int rank = seen_c[r] + warp_excl_scan(ne, lane);
        for (int i = 0; i < 4; ++i)
          if ((eqcb >> i) & 1u) { if (rank < a.kc - gt_c[r]) cb |= 1u << i; ++rank; }
        seen_c[r] += warp_sum(ne);
      }
      // negligible: all below Tn, plus the last (kn - lt_n) keys equal to Tn
      uint32_t nbm = 0u;
      if (a.kn > 0) {
        nbm = ltb;
        if (__any_sync(0xFFFFFFFFu, eqnb != 0u)) {
          const int ne = __popc(eqnb);
          int rank = seen_n[r] + warp_excl_scan(ne, lane);
          for (int i = 0; i < 4; ++i)
            if ((eqnb >> i) & 1u) { if (rank >= eq_n[r] - (a.kn - lt_n[r])) nbm |= 1u << i; ++rank; }
          seen_n[r] += warp_sum(ne);
        }
      }
      crit_bits[r] = cb;
      const size_t row = (size_t)bh * nb + qb0 + r;
      if (j0 < nb) {
        int8_t m[4];
        #pragma unroll
        for (int i = 0; i < 4; ++i) m[i] = ((cb >> i) & 1u) ? 1 : (((nbm >> i) & 1u) ? -1 : 0);
        if (j0 + 3 < nb) {
          if (a.mask) {
            const uint32_t w = (uint32_t)(uint8_t)m[0] | ((uint32_t)(uint8_t)m[1] << 8) |
                               ((uint32_t)(uint8_t)m[2] << 16) | ((uint32_t)(uint8_t)m[3] << 24);
            if (a.mask_vec) *reinterpret_cast<uint32_t*>(a.mask + row * nb + j0) = w;
            else for (int i = 0; i < 4; ++i) a.mask[row * nb + j0 + i] = m[i];
          }
          if (a.m01)
            *reinterpret_cast<uint2*>(a.m01 + row * a.ld_m01 + j0) =
                make_uint2(pack_bf16(m[0] == 0 ? 1.f : 0.f, m[1] == 0 ? 1.f : 0.f),
                           pack_bf16(m[2] == 0 ? 1.f : 0.f, m[3] == 0 ? 1.f : 0.f));
        } else {
          for (int i = 0; i < 4 && j0 + i < nb; ++i) {
            if (a.mask) a.mask[row * nb + j0 + i] = m[i];
            if (a.m01) a.m01[row * a.ld_m01 + j0 + i] = __float2bfloat16_rn(m[i] == 0 ? 1.f : 0.f);
          }
        }
        if (a.scores)
          for (int i = 0; i < 4 && j0 + i < nb; ++i)
            a.scores[row * nb + j0 + i] = expf((okey_value(kk[i]) - row_max[r]) * a.inv_sqrt_d) / row_sum[r];
      }
      if (a.crit_idx) {
        const int nc = __popc(cb);
        int pos = written[r] + warp_excl_scan(nc, lane);
        for (int i = 0; i < 4; ++i)
          if ((cb >> i) & 1u) a.crit_idx[row * a.kc + pos++] = j0 + i;
        written[r] += warp_sum(nc);
      }
    }
    if (lst) {
      const uint32_t u = crit_bits[0] | crit_bits[1];
      const int nu = __popc(u);
      int pos = listed + warp_excl_scan(nu, lane);
      for (int i = 0; i < 4; ++i)
        if ((u >> i) & 1u) {
          const int j = j0 + i;
          if (pos < a.list_cap)
            lst[pos] = (uint32_t)j | ((uint32_t)block_valid_count(a.s, j) << 16) |
                       (((crit_bits[0] >> i) & 1u) << 30) | (((crit_bits[1] >> i) & 1u) << 31);
          ++pos;
        }
      listed += warp_sum(nu);
    }
  }
  for (int r = 0; r < nrows; ++r) {
    const size_t row = (size_t)bh * nb + qb0 + r;
    if (a.m01)
      for (int j = nb + lane; j < a.ld_m01; j += 32) a.m01[row * a.ld_m01 + j] = __float2bfloat16_rn(0.f);
    if (lane == 0 && a.crit_cnt) a.crit_cnt[row] = a.kc;
  }
  if (lst && lane == 0) {
    if (listed > a.list_cap) { atomicCAS(a.status, 0, kErrIndex); listed = a.list_cap; }
    a.list_cnt[(size_t)bh * a.n_pairs + pair] = listed;
  }
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

template <int D>
cudaError_t launch_logits_d(const void* qsplit, const void* ksplit, uint32_t* keys, int BH, int nb, int nbp,
                            int* status, cudaStream_t st) {
  using L = LgLayout<D>;
  CUtensorMap ma, mb;
  const uint64_t dims[3] = {(uint64_t)(3 * D), (uint64_t)nb, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)(3 * D) * 2, (uint64_t)(3 * D) * 2 * nb};
  const uint32_t box[3] = {64, 128, 1};
  if (!make_tile_map(&ma, qsplit, 3, dims, strides, box)) return cudaErrorInvalidValue;
  if (!make_tile_map(&mb, ksplit, 3, dims, strides, box)) return cudaErrorInvalidValue;
  CUtensorMap mk;                                // keys [BH][nb][nbp] uint32, moved as bf16 pairs
  const uint64_t kdims[3] = {(uint64_t)(2 * nbp), (uint64_t)nb, (uint64_t)BH};
  const uint64_t kstrides[2] = {(uint64_t)nbp * 4, (uint64_t)nbp * 4 * nb};
  const uint32_t kbox[3] = {64, 32, 1};
  if (!make_tile_map(&mk, keys, 3, kdims, kstrides, kbox)) return cudaErrorInvalidValue;
  static unsigned long long attr_set = 0;        // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  dim3 grid(nbp / 128, nbp / 128, BH);
  logits_kernel<D><<<grid, 128, L::kBytes, st>>>(ma, mb, mk, nb, nbp, status);
  return cudaGetLastError();
}

}  // namespace

int logits_row_stride(int nb) { return (nb + 127) / 128 * 128; }

cudaError_t launch_logits(const void* qsplit, const void* ksplit, uint32_t* keys, int BH, int nb, int d,
                          int* status, cudaStream_t st) {
  const int nbp = logits_row_stride(nb);
  return d == 128 ? launch_logits_d<128>(qsplit, ksplit, keys, BH, nb, nbp, status, st)
                  : launch_logits_d<64>(qsplit, ksplit, keys, BH, nb, nbp, status, st);
}

cudaError_t launch_classify(const uint32_t* keys, int BH, int nb, int d, int kc, int kn,
                            int8_t* mask, int32_t* crit_idx, int32_t* crit_cnt, __nv_bfloat16* m01, int ld_m01,
                            float* scores, uint32_t* list, int32_t* list_cnt, int list_cap, SeqShape s,
                            int* status, cudaStream_t st) {
  ClsArgs a;
  a.keys = keys; a.nb = nb; a.nbp = logits_row_stride(nb); a.kc = kc; a.kn = kn; a.n_pairs = (nb + 1) / 2;
  a.inv_sqrt_d = (float)(1.0 / sqrt((double)d));
  a.mask = mask; a.mask_vec = (nb % 4 == 0) && (reinterpret_cast<uintptr_t>(mask) % 4 == 0); a.crit_idx = crit_idx; a.crit_cnt = crit_cnt; a.m01 = m01; a.ld_m01 = ld_m01;
  a.scores = scores; a.list = list; a.list_cnt = list_cnt; a.list_cap = list_cap; a.s = s; a.status = status;
  const size_t smem = ((size_t)2 * kClsWarps * a.nbp + kClsWarps * 4 * kMaxCand) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(classify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_pairs + kClsWarps - 1) / kClsWarps, BH);
  classify_kernel<<<grid, kClsWarps * 32, smem, st>>>(a);
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
