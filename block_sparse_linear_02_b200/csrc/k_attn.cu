// k_attn.cu -- block-sparse flash attention on tcgen05 (sm_100a).
//
// Computes, for every 64-token query block i, exact softmax attention over the
// valid keys of a set of 64-token key blocks (SLA page section 3, critical
// branch: "精确的稀疏FlashAttention"; the LVSA page's step-6 formula is the same
// normalised sum).  Optionally adds a gated far-field branch (RoPeSLR page:
// g*local + (1-g)*global, each branch with its own softmax) and an fp32 addend
// (the projected linear branch of SLA: O = O_s + O_l W_proj).
//
// One CTA owns a PAIR of consecutive query blocks (128 query rows = the M of a
// tcgen05 MMA) and walks the union of their key-block sets; each list entry
// carries one flag per half, and a half that does not attend a block masks it
// out.  Warp roles:
//   warp 4  TMA producer: Q once, then K_j/V_j tiles into a 3-stage ring;
//   warp 5  MMA issuer:   S_j = Q K_j^T into one of two TMEM S buffers, then,
//                         once the softmax has written P_j to shared memory,
//                         O += P_j V_j into the TMEM accumulator;
//   warps 0-3 softmax + epilogue: one thread per query row (= TMEM lane);
//                         online softmax in the exp2 domain with lazy
//                         rescaling (the accumulator is rescaled only when the
//                         running max grows by more than 2^8), P written as
//                         bf16 in the 128-byte-swizzled K-major layout the MMA
//                         reads, final normalisation / gate / addend, bf16 store.
#include <cuda_runtime.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

constexpr int kStages = 3;
constexpr uint32_t kColO = 0;      // TMEM columns of the local accumulator (<= 128)
constexpr uint32_t kColS = 128;    // two 64-column S buffers
constexpr uint32_t kColOf = 256;   // far-field accumulator (gated mode)

template <int D>
struct AttnLayout {
  static constexpr int kChunks = D / 64;                 // 64-column (128-byte) chunks
  static constexpr int kQChunk = 128 * 128;              // bytes of one Q chunk (128 rows)
  static constexpr int kKVChunk = 64 * 128;              // bytes of one K/V chunk (64 rows)
  static constexpr int kKVTile = kChunks * kKVChunk;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kChunks * kQChunk;
  static constexpr int kVOff = kKOff + kStages * kKVTile;
  static constexpr int kPOff = kVOff + kStages * kKVTile;
  static constexpr int kBarOff = kPOff + 128 * 128;
  static constexpr int kBytes = kBarOff + 256 + 1024;    // + alignment slack
};

struct AttnKParams {
  int n_pad, seg_len, seg_stride, n_qb, n_kb, n_pairs;
  const uint32_t* list;
  const int32_t* list_cnt;
  int list_cap, list_per_head;
  const float* addend;
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

template <int D, bool TILE, bool GATED>
__global__ void __launch_bounds__(192, 1)
attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKf,
            const __grid_constant__ CUtensorMap tmVf, const AttnKParams p) {
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sK = smem + L::kKOff;
  uint8_t* sV = smem + L::kVOff;
  uint8_t* sP = smem + L::kPOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;
  uint64_t* kv_empty = bars + 1 + 2 * kStages;
  uint64_t* s_full = bars + 1 + 3 * kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_bar = p_full + 1;
  uint64_t* drain = o_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  constexpr uint32_t kTmemCols = GATED ? 512 : 256;

  const uint32_t* list = nullptr;
  int n_local = p.n_kb;
  if (p.list) {
    size_t off = (p.list_per_head ? (size_t)bh * p.n_pairs : 0) + pair;
    list = p.list + off * p.list_cap;
    n_local = p.list_cnt[off];
  }
  const int total = n_local + (GATED ? 1 : 0);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&k_full[s], 1); mbar_init(&v_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(o_bar, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
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
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dK + c * L::kKVChunk, &tmKf, &k_full[s], c * 64, 0, bh);
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(dV + c * L::kKVChunk, &tmVf, &v_full[s], c * 64, 0, bh);
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
      if (*abort_flag) {
        // let the loads already in flight land before the CTA's shared memory is released
        for (int i = (j - kStages > 0 ? j - kStages : 0); i < j; ++i) {
          const int s = i % kStages;
          const long long t0 = clock64();
          while (!mbar_try_wait(&k_full[s], (i / kStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
          while (!mbar_try_wait(&v_full[s], (i / kStages) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
      }
    }
  } else if (warp == 5) {
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
      auto issue_pv = [&](int stage, uint32_t col, bool acc) {
        #pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint64_t a = desc_kmajor(p_addr + kk * 32);
          uint64_t b = desc_mnmajor(v_addr + stage * L::kKVTile + kk * 2048, L::kKVChunk);
          mma_bf16_ss(tmem + col, a, b, idO, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status) && mbar_wait(&k_full[0], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&s_full[0]);
        for (int j = 0; j < total; ++j) {
          if (j + 1 < total) {
            const int s1 = (j + 1) % kStages;
            if (!mbar_wait(&k_full[s1], ((j + 1) / kStages) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_qk(s1, (j + 1) & 1);
            mma_commit(&s_full[(j + 1) & 1]);
          }
          if (!mbar_wait(p_full, j & 1, abort_flag, p.status)) { ok = false; break; }
          const int s = j % kStages;
          if (!mbar_wait(&v_full[s], (j / kStages) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const bool far = GATED && j == n_local;
          issue_pv(s, far ? kColOf : kColO, far ? false : (j > 0));
          mma_commit(o_bar);
          mma_commit(&kv_empty[s]);
        }
      }
      if (!ok) {
        // drain the tensor core before TMEM is released
        mma_commit(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int r = threadIdx.x;              // query row of the pair = TMEM lane
    const int half = r >> 6;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float m_loc = -INFINITY, l_loc = 0.f, m_far = -INFINITY, l_far = 0.f;
    const SeqShape seq{p.n_pad, p.seg_len, p.seg_stride, p.n_kb};
    bool ok = true;
    for (int j = 0; j < total; ++j) {
      const bool far = GATED && j == n_local;
      const int sb = j & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag, p.status))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(lane_addr + kColS + sb * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(lane_addr + kColS + sb * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      int nvalid = 64;
      bool attend = true;
      if (!far) {
        const uint32_t e = list ? list[j] : ((uint32_t)j | 0xC0000000u);
        attend = (e >> (30 + half)) & 1u;
        if (!TILE) nvalid = block_valid_count(seq, (int)(e & 0x3FFFFFFFu));
      }
      float mx = -INFINITY;
      #pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float x = (attend && c < nvalid) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
        sr[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      float& m = far ? m_far : m_loc;
      float& l = far ? l_far : l_loc;
      const float m_new = fmaxf(m, mx);
      const bool need = m_new > m + 8.f;
      float factor = 1.f;
      if (need) { factor = exp2f(m - m_new); l *= factor; m = m_new; }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float rowsum = 0.f;
      uint32_t packed[32];
      #pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = exp2f(__uint_as_float(sr[c]) - mu);
        const float p1 = exp2f(__uint_as_float(sr[c + 1]) - mu);
        rowsum += p0 + p1;
        packed[c >> 1] = pack_bf16(p0, p1);
      }
      l += rowsum;
      // P buffer and accumulator are free once P_{j-1} V_{j-1} has completed
      if (j > 0) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(o_bar, (j - 1) & 1, abort_flag, p.status))) { ok = false; break; }
        tc_fence_after();
      }
      if (!far && j > 0 && __any_sync(0xFFFFFFFFu, need)) {
        #pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + cc * 32, o);
          tmem_wait_ld();
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(lane_addr + kColO + cc * 32, o);
        }
        tmem_wait_st();
      }
      #pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint4 val = make_uint4(packed[4 * c8], packed[4 * c8 + 1], packed[4 * c8 + 2], packed[4 * c8 + 3]);
        *reinterpret_cast<uint4*>(sP + sw128_offset(r, c8)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && total > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(o_bar, (total - 1) & 1, abort_flag, p.status));
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();

    // ---- epilogue: row r of the pair -> token index
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
    const float inv_l = (l_loc > 0.f) ? 1.f / l_loc : 0.f;
    const float inv_lf = (l_far > 0.f) ? 1.f / l_far : 0.f;
    const size_t row_off = ((size_t)bh * p.n_pad + (row_exists ? tok : 0)) * D;
    const bool read_tmem = ok && total > 0;      // CTA-uniform
    #pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      float v[32];
      if (read_tmem) {
        tmem_ld32(lane_addr + kColO + cc * 32, o);
        tmem_wait_ld();
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv_l;
        if (GATED) {
          tmem_ld32(lane_addr + kColOf + cc * 32, o);
          tmem_wait_ld();
          #pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = p.gate * v[i] + (1.f - p.gate) * (__uint_as_float(o[i]) * inv_lf);
        }
      } else {
        #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (!row_exists) continue;
      if (valid && p.addend) {
        const float4* ad = reinterpret_cast<const float4*>(p.addend + row_off + cc * 32);
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
          float4 a4 = __ldg(ad + i);
          v[4 * i] += a4.x; v[4 * i + 1] += a4.y; v[4 * i + 2] += a4.z; v[4 * i + 3] += a4.w;
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out + row_off + cc * 32);
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        if (valid) {
          w = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                         pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
        } else {
          w = make_uint4(0, 0, 0, 0);
        }
        dst[i] = w;
      }
    }
    if (p.lse && row_exists) {
      float val = 0.f;
      if (valid) val = (l_loc > 0.f) ? (m_loc + log2f(l_loc)) * 0.69314718055994531f : -INFINITY;
      p.lse[(size_t)bh * p.n_pad + tok] = val;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool TILE, bool GATED>
cudaError_t launch_variant(const AttnArgs& a, const CUtensorMap* maps, const AttnKParams& kp, cudaStream_t st) {
  using L = AttnLayout<D>;
  auto kern = attn_kernel<D, TILE, GATED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_pairs, a.BH);
  kern<<<grid, 192, L::kBytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], kp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  const int D = a.d;
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
  if (a.gated) {
    const uint64_t dims[3] = {(uint64_t)D, 64, (uint64_t)a.BH};
    const uint64_t strides[2] = {rowb, rowb * 64};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tile_map(&maps[3], a.kf, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[4], a.vf, 3, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  AttnKParams kp;
  kp.n_pad = a.s.n_pad; kp.seg_len = a.s.seg_len; kp.seg_stride = a.s.seg_stride;
  kp.n_qb = a.n_qb; kp.n_kb = a.n_kb; kp.n_pairs = a.n_pairs;
  kp.list = a.list; kp.list_cnt = a.list_cnt; kp.list_cap = a.list_cap; kp.list_per_head = a.list_per_head;
  kp.addend = a.addend; kp.out = reinterpret_cast<__nv_bfloat16*>(a.out); kp.lse = a.lse;
  kp.F = a.F; kp.Hh = a.Hh; kp.Ww = a.Ww;
  kp.TF = a.tile3d ? a.F / 4 : 1; kp.TH = a.tile3d ? a.Hh / 4 : 1; kp.TW = a.tile3d ? a.Ww / 4 : 1;
  kp.gate = a.gate;
  kp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  kp.status = a.status;
  if (D == 128) {
    if (a.tile3d) return a.gated ? launch_variant<128, true, true>(a, maps, kp, st) : launch_variant<128, true, false>(a, maps, kp, st);
    return a.gated ? launch_variant<128, false, true>(a, maps, kp, st) : launch_variant<128, false, false>(a, maps, kp, st);
  }
  if (a.tile3d) return a.gated ? launch_variant<64, true, true>(a, maps, kp, st) : launch_variant<64, true, false>(a, maps, kp, st);
  return a.gated ? launch_variant<64, false, true>(a, maps, kp, st) : launch_variant<64, false, false>(a, maps, kp, st);
}

}  // namespace slr
