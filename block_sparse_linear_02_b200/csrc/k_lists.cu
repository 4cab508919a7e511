// k_lists.cu -- key-block lists for the attention kernel.
//
// The attention kernel handles query blocks in pairs (128 rows = one tcgen05
// M tile).  pair_lists_kernel turns per-query-block key-block sets into one
// ascending list per pair: each entry is a key block of the union of the two
// sets with its number of valid keys, tagged with which half attends it.  Sets come from
//   - explicit per-query-block lists (SLA's critical lists or a caller's),
//   - LVSA frame sets A(t) expanded to the key blocks of each frame (rainbus
//     page, step 6: all tokens of the attended frames),
//   - the 3x3x3 tile neighbourhood of the RoPeSLR local branch (aixinbiao page).
// Membership is collected in two shared-memory bitmaps (so a set's order and
// duplicates do not matter) and compacted by one warp in index order.
//
// lvsa_sets_kernel builds A(t) for every frame with the routine in lvsa_sets.cuh.
#include <cuda_runtime.h>

#include "launch.h"
#include "lvsa_sets.cuh"
#include "sm100.cuh"

namespace slr {
namespace {

constexpr int kWords = kMaxKeyBlocks / 32;

__global__ void __launch_bounds__(256)
pair_lists_kernel(const ListArgs a) {
  __shared__ uint32_t bm[2][kWords];
  const int pair = blockIdx.x, head = blockIdx.y;
  const int nwords = (a.n_kb + 31) / 32;
  for (int i = threadIdx.x; i < 2 * kWords; i += blockDim.x) (&bm[0][0])[i] = 0u;
  __syncthreads();
  for (int half = 0; half < 2; ++half) {
    const int qb = 2 * pair + half;
    if (qb >= a.n_qb) continue;
    if (a.mode == kListExplicit) {
      const size_t row = (size_t)head * a.n_qb + qb;
      int cnt = a.kv_cnt[row];
      if (cnt < 0 || cnt > a.kv_max) {
        if (threadIdx.x == 0) atomicCAS(a.status, 0, kErrIndex);
        cnt = cnt < 0 ? 0 : a.kv_max;
      }
      const int32_t* idx = a.kv_idx + row * a.kv_max;
      for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
        const int j = idx[e];
        if (j < 0 || j >= a.n_kb) { atomicCAS(a.status, 0, kErrIndex); continue; }
        atomicOr(&bm[half][j >> 5], 1u << (j & 31));
      }
    } else if (a.mode == kListLvsa) {
      const int t = qb / a.blocks_per_frame;
      int cnt = a.set_cnt[t];
      if (cnt < 0) {
        if (threadIdx.x == 0) atomicCAS(a.status, 0, kErrIndex);
        cnt = 0;
      }
      for (int e = threadIdx.x; e < cnt * a.blocks_per_frame; e += blockDim.x) {
        const int f = a.sets[(size_t)t * a.set_cap + e / a.blocks_per_frame];
        const int j = f * a.blocks_per_frame + e % a.blocks_per_frame;
        if (j < 0 || j >= a.n_kb) { atomicCAS(a.status, 0, kErrIndex); continue; }
        atomicOr(&bm[half][j >> 5], 1u << (j & 31));
      }
    } else {  // tile neighbourhood
      const int tf = qb % a.TF, tw = (qb / a.TF) % a.TW, th = (qb / a.TF) / a.TW;
      const int sf = 2 * a.rad[0] + 1, sh = 2 * a.rad[1] + 1, sw = 2 * a.rad[2] + 1;
      for (int e = threadIdx.x; e < sf * sh * sw; e += blockDim.x) {
        const int nf = tf + e / (sh * sw) - a.rad[0];
        const int nh = th + (e / sw) % sh - a.rad[1];
        const int nw = tw + e % sw - a.rad[2];
        if (nf < 0 || nf >= a.TF || nh < 0 || nh >= a.TH || nw < 0 || nw >= a.TW) continue;
        const int j = (nh * a.TW + nw) * a.TF + nf;
        atomicOr(&bm[half][j >> 5], 1u << (j & 31));
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t* out = a.list + ((size_t)head * a.n_pairs + pair) * a.cap;
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t b0 = w < nwords ? bm[0][w] : 0u;
      const uint32_t b1 = w < nwords ? bm[1][w] : 0u;
      uint32_t u = b0 | b1;
      const int c = __popc(u);
      int incl = c;
      #pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - c;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        if (pos < a.cap) {
          const int j = w * 32 + bit;
          const uint32_t nv = a.mode == kListTile3d ? 64u : (uint32_t)block_valid_count(a.s, j);
          out[pos] = (uint32_t)j | (nv << 16) | (((b0 >> bit) & 1u) << 30) | (((b1 >> bit) & 1u) << 31);
        }
        ++pos;
      }
      base += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
      if (base > a.cap) { atomicCAS(a.status, 0, kErrIndex); base = a.cap; }
      a.list_cnt[(size_t)head * a.n_pairs + pair] = base;
    }
  }
}

__global__ void lvsa_sets_kernel(int T, int C, int W, int step, int32_t* sets, int32_t* counts, int cap) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  counts[t] = lvsa_attention_set(T, C, W, step, t, sets + (size_t)t * cap, cap);
}

}  // namespace

cudaError_t launch_pair_lists(const ListArgs& a, int heads, cudaStream_t st) {
  dim3 grid(a.n_pairs, heads);
  pair_lists_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_lvsa_sets(int T, int C, int W, int step, int32_t* sets, int32_t* counts, int cap,
                             cudaStream_t st) {
  lvsa_sets_kernel<<<(T + 127) / 128, 128, 0, st>>>(T, C, W, step, sets, counts, cap);
  return cudaGetLastError();
}

}  // namespace slr
