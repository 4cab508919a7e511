// launch.h -- host-side launch interface between the C ABI (slr_api.cu) and the
// kernels (k_*.cu).  Every launcher queues its kernels on `stream` and returns a
// cudaError_t from the launch; none synchronises.
#pragma once

#include <cuda_runtime.h>
#include <cuda.h>

#include "../../include/slr.h"   // the SLR_PHI_* feature-map codes the kernels take
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace slr {

// ------------------------------------------------------------ tensor maps
// A tile map over a bf16 tensor whose innermost dimension is contiguous.
// dims[0] is the innermost extent (elements), strides are in bytes for dims 1..rank-1.
// swizzle_bytes: 128 (the default), 64, 32 or 0 (none); the box's inner extent in
// bytes must not exceed it when it is not 0.
bool make_tile_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes = 128);

// ------------------------------------------------------------ pooling (k_pool.cu)
// Means of the valid tokens of every 64-token block of q and k, each written as a
// bf16 pair hi + lo: rows [BH][Nb][3d], [qh | qh | ql] for q and [kh | kl | kh] for k.
// With phi_q non-null, also phi(q) in bf16 [BH][N_pad][d] (pad tokens 0); phi is
// SLR_PHI_ELU1 (elu(q) + 1) or SLR_PHI_SOFTMAX (softmax of each row over its d channels).
cudaError_t launch_pool_means(const void* q, const void* k, void* qsplit, void* ksplit, void* phi_q, int phi,
                              int BH, int d, SeqShape s, cudaStream_t st);

// ------------------------------------------------------------ tile layouts (k_far.cu)
// Tile-major order of a raster (F, Hh, Ww) sequence (F, Hh, Ww multiples of 4): 4x4x4
// tile (th * TW + tw) * TF + tf takes rows [64 tile, 64 tile + 64), its tokens in (f, h, w)
// raster order inside the tile.  launch_tile_major copies K and V into that order
// (bf16 [BH][F*Hh*Ww][d] each).
cudaError_t launch_tile_major(const void* k, const void* v, void* kt, void* vt, int BH, int d, int F, int Hh,
                              int Ww, cudaStream_t st);

// The RoPeSLR far-field pass: K and V written in tile-major order into kt and vt, and
// their means over cells of (cf, ch, cw) tokens into kf and vf (bf16 [BH][ncells][d], cells
// in raster order of the cell grid), through fp32 row sums in `part`
// (far_partial_bytes).  With rope = 1, q and k are first rotated by the 3-D rotary
// embedding (base 10000, channel pairs split frame / height / width; the cos / sin table
// in `tab`, far_rope_table_bytes) and the rotated q is written, in raster order, into qr.
// A raster row of Ww tokens passes through shared memory: Ww * d * 2 <= kFarRowBytesMax.
constexpr size_t kFarRowBytesMax = 96 * 1024;
size_t far_rope_table_bytes(int d, int F, int Hh, int Ww);
size_t far_partial_bytes(int BH, int d, int F, int Hh, int Ww, int cw);
cudaError_t launch_far_field(const void* q, const void* k, const void* v, void* qr, void* kt, void* vt, void* kf,
                             void* vf, void* tab, void* part, int BH, int d, int F, int Hh, int Ww, int cf, int ch,
                             int cw, int rope, cudaStream_t st);

// ------------------------------------------------------------ classification (k_classify.cu)
// Row stride (entries) of the logit-key matrix: Nb rounded up to 128.
int logits_row_stride(int nb);

// keys[bh][i][j] = order-preserving uint32 key of the logit qbar_i . kbar_j (from the
// split rows of launch_pool_means), row stride logits_row_stride(nb), pad entries 0.
cudaError_t launch_logits(const void* qsplit, const void* ksplit, uint32_t* keys, int BH, int nb, int d,
                          int* status, cudaStream_t st);

// Labels per row from the logit keys (top kc -> 1, bottom kn -> -1, rest 0, ties to
// the lower index) and the outputs, each optional (nullptr = skip): mask
// [BH][nb][nb]; crit_idx [BH][nb][kc] ascending and crit_cnt [BH][nb]; the marginal
// indicator m01 (bf16 1/0, row stride ld_m01, pad columns 0); P_c =
// softmax(logits / sqrt(d)) in fp32; pair lists [BH][(nb+1)/2][list_cap] of the
// union of the critical sets of query blocks 2p and 2p+1 (entry layout below) with
// counts list_cnt [BH][(nb+1)/2].
cudaError_t launch_classify(const uint32_t* keys, int BH, int nb, int d, int kc, int kn,
                            int8_t* mask, int32_t* crit_idx, int32_t* crit_cnt, __nv_bfloat16* m01, int ld_m01,
                            float* scores, uint32_t* list, int32_t* list_cnt, int list_cap, SeqShape s,
                            int* status, cudaStream_t st);

// m01 = (mask == 0) as bf16 with row stride ld_m01 (pad columns zeroed).
cudaError_t launch_mask_to_m01(const int8_t* mask, __nv_bfloat16* m01, int BH, int nb, int ld_m01,
                               cudaStream_t st);

// ------------------------------------------------------------ block lists (k_lists.cu)
// Entries of a pair list: key block index in bits [0,16), its number of valid keys
// in bits [16,23), bit 30 = the first query block of the pair attends it, bit 31 =
// the second does.
enum ListMode { kListExplicit = 0, kListLvsa = 1, kListTile3d = 2 };

struct ListArgs {
  int mode;
  int n_qb, n_kb, n_pairs, cap;
  // explicit
  const int32_t* kv_idx;   // [BH][n_qb][kv_max]
  const int32_t* kv_cnt;   // [BH][n_qb]
  int kv_max;
  // lvsa
  const int32_t* sets;     // [T][set_cap]
  const int32_t* set_cnt;  // [T]
  int set_cap, blocks_per_frame;
  // tile3d: tile grid (TF, TH, TW), tile id = (th*TW + tw)*TF + tf; a key tile is a
  // neighbour when it is within rad[0] / rad[1] / rad[2] tiles on the frame / height /
  // width axis
  int TF, TH, TW, rad[3];
  SeqShape s;              // token layout (valid-key counts of linear blocks)
  uint32_t* list;          // [heads][n_pairs][cap]
  int32_t* list_cnt;       // [heads][n_pairs]
  int* status;
};
cudaError_t launch_pair_lists(const ListArgs& a, int heads, cudaStream_t st);

// LVSA attention sets on the device (one thread per frame).
cudaError_t launch_lvsa_sets(int T, int C, int W, int step, int32_t* sets, int32_t* counts, int cap,
                             cudaStream_t st);

// ------------------------------------------------------------ attention (k_attn.cu)
struct AttnArgs {
  const void* q; const void* k; const void* v;
  const void* kf; const void* vf;      // far-field pooled K/V, bf16 [BH][64][d] (gated mode)
  int BH, d;
  SeqShape s;
  int n_qb, n_kb, n_pairs;
  const uint32_t* list;                // null = dense
  const int32_t* list_cnt;
  int list_cap, list_per_head;         // list_per_head = 0 when one list serves all heads
  const __nv_bfloat16* Hs;             // SLA linear branch: [BH][n_qb][(d+1)][d] rows [H_i'^T ; Z_i], or null
  const void* phi_q;                   // SLA linear branch: phi(q) bf16 [BH][n_pad][d] (with Hs)
  void* out;                           // bf16 [BH][n_pad][d]
  float* lse;                          // fp32 [BH][n_pad] or null
  int tile3d;                          // 1: blocks are 4x4x4 tiles of raster (F, Hh, Ww)
  int F, Hh, Ww;
  int gated;                           // 1: add the far-field branch and gate
  float gate;
  int* status;
  int* tile_counter;                   // one int of scratch, zeroed by launch_attention on the stream
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st);

// ------------------------------------------------------------ marginal branch (k_marginal.cu)
// h[bh][j] = [ (phi(K_j)^T V_j W)^T (d rows of d) ; z_j (1 row) ] in bf16, [BH][nb][(d+1)*d];
// W = w_proj (bf16 [d][d]) or the identity when w_proj is null.
cudaError_t launch_key_states(const void* k, const void* v, const void* w_proj, __nv_bfloat16* h, int phi, int BH,
                              int d, SeqShape s, int* status, cudaStream_t st);

// Hs[bh][i] = sum_j m01[bh][i][j] * h[bh][j]  (bf16 out, fp32 accumulate), [BH][nb][(d+1)*d].
cudaError_t launch_reduce_states(const __nv_bfloat16* m01, int ld_m01, const __nv_bfloat16* h,
                                 __nv_bfloat16* Hs, int BH, int nb, int d, int* status, cudaStream_t st);

// o_lin[bh][t] = phi(q_t) H_i' / (phi(q_t).Z_i) for every valid token t of block i (0 for pads).
// ------------------------------------------------------------ SVOO co-clustering (k_svoo.cu)
// Cluster counts are padded to Cp = the power of two >= max(C, 32); C <= kSvooMaxClusters.
// Centres are fp32 [BH][Cp][d]; ub bf16 [BH][Cp][3d] and bias fp32 [BH][Cp] hold the metric
// of the assigning side; labels and perm are int32 [BH][n_pad]; counts and offs int32
// [BH][svoo_sort_chunks(n_pad)][C + 1] (counts zero before the first assignment; the sort
// clears them again); start int32 [BH][C + 2].
constexpr int kSvooMaxClusters = 128;
int svoo_padded_clusters(int C);
int svoo_sort_chunks(int n_pad);
// centres[n] = x[anchor[n]] (an anchor that is not a valid token sets SLR_ERR_INDEX)
cudaError_t launch_svoo_anchors(const void* x, const int32_t* anchor, float* centres, int C, int BH, int d,
                                SeqShape s, int* status, cudaStream_t st);
// labels of the tokens of x: the own centre (of C_own) whose affinity vector against the
// C_other centres of the other side is nearest (pads: C_own); label histogram into counts
cudaError_t launch_svoo_assign(const void* x, const float* other, int C_other, float* own, int C_own,
                               __nv_bfloat16* ub, float* bias, int32_t* labels, int32_t* counts, int BH, int d,
                               SeqShape s, int* status, cudaStream_t st);
// the stable order of the labels: perm (position -> token), the cluster starts and the
// piece offsets of the update (poff int32 [BH][C + 1])
cudaError_t launch_svoo_sort(const int32_t* labels, int32_t* counts, int32_t* offs, int32_t* start, int32_t* poff,
                             int32_t* perm, int C, int BH, SeqShape s, cudaStream_t st);
// centres = means of their tokens (an empty cluster keeps its centre), through fp64 piece
// sums part [BH][svoo_max_pieces(n_pad, C)][d]
int svoo_max_pieces(int n_pad, int C);
cudaError_t launch_svoo_update(const void* x, const int32_t* perm, const int32_t* start, const int32_t* poff,
                               double* part, float* centres, int C, int BH, int d, SeqShape s, cudaStream_t st);
// qp[p] = q[q_perm[p]], kp[p] = k[k_perm[p]], vp[p] = v[k_perm[p]] (bf16 rows of d)
cudaError_t launch_svoo_gather(const void* q, const void* k, const void* v, const int32_t* q_perm,
                               const int32_t* k_perm, void* qp, void* kp, void* vp, int BH, int d, int n_pad,
                               int* status, cudaStream_t st);
// out[q_perm[p]] = src[p]
cudaError_t launch_svoo_scatter_rows(const void* src, const int32_t* q_perm, void* out, int BH, int d, int n_pad,
                                     int* status, cudaStream_t st);

// ------------------------------------------------------------ no-workspace call (slr_noalloc.cu)
// Reads and clears the status word of the static scratch on the current device.
int noalloc_check_status(void* stream);   // an slr_status value

cudaError_t launch_linear_apply(const void* q, const __nv_bfloat16* Hs, float* o_lin, int phi, int BH, int d,
                                SeqShape s, int* status, cudaStream_t st);

}  // namespace slr
