// common.cuh -- shapes, status codes and small helpers shared by the kernels
// and the host-side entry points of libslr.
#pragma once

#include <stdint.h>

namespace slr {

// Device status codes (the negated public slr_status values).
constexpr int kErrTimeout = 5;   // SLR_ERR_TIMEOUT
constexpr int kErrIndex = 6;     // SLR_ERR_INDEX

constexpr int kBlock = 64;        // tokens per query / key block
constexpr int kMaxKeyBlocks = 8192;
constexpr int kMaxClassifyBlocks = 4096;

// Token layout of one (b, h) sequence: n_seg segments of seg_stride tokens,
// the first seg_len of which are valid.
struct SeqShape {
  int n_pad;       // n_seg * seg_stride
  int seg_len;
  int seg_stride;
  int n_blocks;    // n_pad / 64
};

// Number of valid tokens in 64-token block j (every block holds at least one).
__host__ __device__ __forceinline__ int block_valid_count(const SeqShape& s, int j) {
  int off = (j * kBlock) % s.seg_stride;
  int v = s.seg_len - off;
  return v < 0 ? 0 : (v > kBlock ? kBlock : v);
}

__host__ __device__ __forceinline__ bool token_valid(const SeqShape& s, int t) {
  return t < s.n_pad && (t % s.seg_stride) < s.seg_len;
}

}  // namespace slr
