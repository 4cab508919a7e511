/*
 * slr.h -- C ABI of libslr: block-sparse + linear attention over the
 * (frame x height x width) token sequence of a video diffusion transformer,
 * hand-written for NVIDIA B200 (sm_100a).
 *
 * The operations follow these source write-ups:
 *  - SLA (Sparse-Linear Attention, arXiv 2509.24006), techwalker page
 *    "清华大学破解视频生成卡顿难题", section 3 "SLA方法的核心机制";
 *  - LVSA (arXiv 2605.31057), rainbus paper digest, sections "核心方法" and
 *    "方法步骤详情";
 *  - RoPeSLR (arXiv 2605.20659), aixinbiao blog, section "稀疏邻域加低秩远场";
 *  - VORTA (arXiv 2505.18809), zhaoyang97 paper notes, section "方法详解";
 *  - SVOO (arXiv 2603.18636), gist.science summary, section 3.
 *
 * Conventions shared by every compute entry point
 * ------------------------------------------------
 *  - Tensors q, k, v, out are caller-owned DEVICE pointers to bf16 arrays laid
 *    out [B][H][N_pad][d], contiguous, 16-byte aligned.  N_pad =
 *    n_seg * seg_stride; inside each segment the first seg_len tokens are
 *    valid and the rest are padding.  Pad keys are excluded from every sum;
 *    pad query rows of every output are written as 0.
 *  - Each call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  No call synchronises, allocates or
 *    frees memory.  Scratch memory is the caller's `ws` (device, 256-byte
 *    aligned) of at least slr_workspace_bytes(...) bytes; its first 256 bytes
 *    hold the device status word, reset at the start of every call.
 *  - Return value: SLR_OK when the launches were queued.  Argument errors are
 *    detected on the host before anything is launched.  Errors found by the
 *    device (an out-of-range index in a caller's list, a bounded wait that
 *    expired) are written to the status word and returned by
 *    slr_check_status().
 *  - Supported shapes: d in {64, 128}; block == 64; seg_stride a multiple of
 *    64; seg_len in (seg_stride - 64, seg_stride] so that every 64-token block
 *    holds at least one valid token; N_pad / 64 <= 8192 key blocks (4096 for
 *    the classifying calls).
 */
#ifndef SLR_H
#define SLR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int slr_status;
#define SLR_OK               0
#define SLR_ERR_ARG         (-1)  /* null/misaligned pointer, bad size, inconsistent fractions   */
#define SLR_ERR_UNSUPPORTED (-2)  /* a shape outside the supported set above                      */
#define SLR_ERR_WORKSPACE   (-3)  /* ws_bytes below slr_workspace_bytes() or ws misaligned        */
#define SLR_ERR_CUDA        (-4)  /* a CUDA runtime call or kernel launch failed                  */
#define SLR_ERR_TIMEOUT     (-5)  /* device: a bounded wait expired; the kernel exited cleanly     */
#define SLR_ERR_INDEX       (-6)  /* device: a caller-supplied block index was out of range        */

/* Sequence descriptor: B batches, H heads, head size d, 64-token blocks, and
 * n_seg segments of seg_stride tokens of which the first seg_len are valid. */
typedef struct {
    int B, H, d, block;
    int n_seg, seg_len, seg_stride;
} slr_seq;

/* Feature map of the linear branch; SLA page section 3 names phi, and the
 * plainest reading used here is phi(x) = elu(x) + 1.  The page later reports that
 * a softmax activation works better there; SLR_PHI_SOFTMAX reads it as the softmax
 * of each q and k row over its d channels. */
#define SLR_PHI_ELU1 0
#define SLR_PHI_SOFTMAX 1

/* External block masks for slr_frame_mask_attn. */
#define SLR_MASK_LVSA   1
#define SLR_MASK_TILE3D 2
#define SLR_MASK_STA    3
typedef struct {
    int kind;                 /* SLR_MASK_LVSA, SLR_MASK_TILE3D or SLR_MASK_STA                */
    /* LVSA (rainbus page, "方法步骤详情" steps 1-6): frames are the n_seg segments, T == n_seg */
    int T, C, W, step;        /* frames, budget, window half-width, denoising step s            */
    /* TILE3D (aixinbiao page) and STA (VORTA page): raster (F, Hh, Ww) tokens,
       F*Hh*Ww == N_pad, n_seg == 1                                                            */
    int F, Hh, Ww;
    int tile[3];              /* token tile, must be {4, 4, 4}                                  */
    int radius;               /* Chebyshev tile radius of the local neighbourhood (1 -> 3x3x3)  */
    int cell[3];              /* far-field pooling cell; the cell grid must hold 64 cells       */
    float gate;               /* g in g*local + (1-g)*global                                    */
    int rope;                 /* TILE3D: 1 = rotate q and k by the 3-D rotary embedding first
                                 (aixinbiao page: the neighbourhood branch encodes relative
                                 position with RoPE); 0 = take q and k as given.  LVSA, STA: 0 */
    int window[3];            /* STA: window (frame, height, width) in tokens, each an odd
                                 multiple of the tile size 4                                   */
} slr_mask_desc;

/* Percentile parameters for the classifying calls (params of slr_workspace_bytes). */
typedef struct {
    float crit_frac;          /* fraction of key blocks per query-block row labelled critical   */
    float negl_frac;          /* fraction labelled negligible                                   */
} slr_fracs;

/* Operation codes for slr_workspace_bytes. */
#define SLR_OP_POOL_CLASSIFY   1   /* params: const slr_fracs*                     */
#define SLR_OP_BLOCK_SPARSE    2   /* params: const int* kv_max                    */
#define SLR_OP_LINEAR_MARGINAL 3   /* params: unused (NULL)                        */
#define SLR_OP_SPARSE_LINEAR   4   /* params: const slr_fracs*                     */
#define SLR_OP_FRAME_MASK      5   /* params: const slr_mask_desc*                 */
#define SLR_OP_SVOO_COCLUSTER  6   /* params: const int[2] {n_qc, n_kc}            */
#define SLR_OP_SVOO_ATTN       7   /* params: const float* keep_frac               */

/* ------------------------------------------------------------------ compute */

/*
 * slr_pool_classify -- SLA page section 3, first two paragraphs: mean-pool Q
 * and K per 64-token block (valid tokens only), form the compressed scores
 * P_c = softmax(pool(Q) pool(K)^T / sqrt(d)) per (b, h, query block), and label
 * each key block of a row critical (1, the kc highest), negligible (-1, the kn
 * lowest) or marginal (0), ranking by score descending then index ascending.
 * kc = max(1, ceil(crit_frac*Nkb)), kn = floor(negl_frac*Nkb), kc+kn <= Nkb
 * (see slr_block_counts).
 * Precision: each block sum is exact (fp64 over at most 64 bf16 values) and the
 * mean is kept as a bf16 pair hi + lo (16 significant bits); the logits are
 * formed on the tensor cores from those pairs (the products hi.hi, hi.lo and
 * lo.hi in bf16 with fp32 accumulation; lo.lo, ~2^-16 relative, is dropped).
 * P_c is then within ~1e-8 of its fp64 value (the tests bound it by 1e-6), so
 * a label can differ from an exact-arithmetic ranking only for a pair whose
 * P_c lies that close to its row's threshold; row counts are always exact and
 * exact ties go to the lower key-block index.
 *
 *   q, k       bf16 [B][H][N_pad][d] device, read only
 *   mask       int8 [B][H][Nb][Nb] device, written
 *   crit_idx   int32 [B][H][Nb][kc] device, written: the critical key blocks of
 *              each row, ascending
 *   crit_cnt   int32 [B][H][Nb] device, written (always kc)
 *   scores_opt float [B][H][Nb][Nb] device or NULL: P_c rounded to fp32
 * Requires 0 <= crit_frac, negl_frac <= 1.
 */
slr_status slr_pool_classify(const void* q, const void* k, const slr_seq* seq,
                             float crit_frac, float negl_frac,
                             int8_t* mask, int32_t* crit_idx, int32_t* crit_cnt,
                             float* scores_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * slr_block_sparse_attn -- exact softmax attention of every query block over
 * a caller-given set of key blocks (SLA page section 3, critical branch; the
 * LVSA page's step-6 formula is the same normalised sum).  Each query of query
 * block i attends every valid key of the key blocks kv_idx[b][h][i][0..cnt-1]
 * (a set: order is irrelevant, duplicates count once), with scale 1/sqrt(d).
 * A query block with an empty set gets 0.  kv_idx == NULL selects the dense
 * mode: every query block attends every key block.
 *
 *   kv_idx   int32 [B][H][Nb][kv_max] device or NULL; entries in [0, Nb)
 *   kv_cnt   int32 [B][H][Nb] device (ignored when kv_idx is NULL); 0..kv_max
 *   o        bf16 [B][H][N_pad][d] device, written
 *   lse_opt  float [B][H][N_pad] device or NULL: natural-log log-sum-exp of the
 *            scaled logits per query (-inf for a query with no key, 0 for pads)
 * An out-of-range index sets SLR_ERR_INDEX in the status word.
 */
slr_status slr_block_sparse_attn(const void* q, const void* k, const void* v, const slr_seq* seq,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, int kv_max,
                                 void* o, float* lse_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * slr_linear_marginal -- the SLA linear branch (SLA page section 3, marginal
 * weights): per key block j precompute h_j = phi(K_j)^T V_j and
 * z_j = sum_t phi(K_j,t) over valid tokens; per query block i reduce
 * H_i = sum_{mask[i][j]==0} h_j, Z_i likewise, and output
 * O_l,t = phi(q_t) H_i / (phi(q_t) . Z_i) (0 if row i has no marginal block),
 * optionally multiplied on the right by W_proj (SLA page, projection paragraph).
 *
 *   mask       int8 [B][H][Nb][Nb] device: 0 = marginal, anything else = not
 *   phi        SLR_PHI_ELU1 or SLR_PHI_SOFTMAX
 *   w_proj_opt bf16 [d][d] device or NULL (NULL = no projection)
 *   o_lin      float [B][H][N_pad][d] device, written
 */
slr_status slr_linear_marginal(const void* q, const void* k, const void* v, const slr_seq* seq,
                               const int8_t* mask, int phi, const void* w_proj_opt,
                               float* o_lin, void* ws, size_t ws_bytes, void* stream);

/*
 * slr_sparse_linear_attn -- the full SLA forward (SLA page section 3):
 * slr_pool_classify, then O = O_s + O_l W_proj with O_s the critical-branch
 * softmax attention and O_l the marginal-branch linear attention; negligible
 * blocks are skipped.  crit_frac = 1, negl_frac = 0 is the dense mode: no
 * classification and no linear branch, full softmax attention.
 *
 *   w_proj        bf16 [d][d] device (may be NULL in dense mode)
 *   out           bf16 [B][H][N_pad][d] device, written
 *   mask_out_opt  int8 [B][H][Nb][Nb] device or NULL: the labels used
 */
slr_status slr_sparse_linear_attn(const void* q, const void* k, const void* v, const void* w_proj,
                                  const slr_seq* seq, float crit_frac, float negl_frac, int phi,
                                  void* out, int8_t* mask_out_opt,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * slr_frame_mask_attn -- attention under an externally defined block mask.
 *  SLR_MASK_LVSA (rainbus page, steps 1-6): frames are the n_seg segments
 *    (T == n_seg).  For denoising step `step` the attention sets
 *    A(t) = G_s u W(t) are built on the device (the same routine as
 *    slr_lvsa_attention_sets) and every query of frame t attends, with one
 *    softmax, every valid key of the frames of A(t).
 *  SLR_MASK_TILE3D (aixinbiao page): q, k, v are in raster (F, Hh, Ww) order;
 *    every query attends, with one softmax, all tokens of the 4x4x4 tiles
 *    within Chebyshev tile distance `radius` of its own tile (clipped at the
 *    borders), and separately, with its own softmax, 64 far-field tokens made
 *    by mean-pooling K and V over `cell`-sized cells; the output is
 *    gate*local + (1-gate)*far.  With rope = 1, q and k are first rotated by the
 *    3-D rotary embedding (base 10000; with P = d/2 channel pairs, the height and
 *    width axes take floor(P/3) consecutive pairs each after the frame axis's
 *    P - 2 floor(P/3); pair i of an axis group of n pairs turns by
 *    coordinate * 10000^(-i/n)), for both branches: the far field pools the
 *    rotated K; the rotated q is kept in the workspace (B*H*N_pad*d bf16).
 *  SLR_MASK_STA (VORTA paper notes, section 方法详解, design 1: 3-D sliding tile
 *    attention, M = {j in (tau(i) - w, tau(i) + w]} with tau the centre of the
 *    position's tile): q, k, v are in raster (F, Hh, Ww) order, tiles are
 *    4x4x4 tokens, and a query attends, with one softmax, every key whose tile
 *    centre lies, on every axis, in (tau(query) - W/2, tau(query) + W/2] for
 *    that axis's window W = `window` -- with W = (2r+1)*4 the tiles within r
 *    tiles of the query's tile, clipped at the borders.  No far field, no gate.
 *  TILE3D needs Ww * d * 2 <= 96 KB (a raster row of K or V passes through
 *    shared memory in the far-field pass), else SLR_ERR_UNSUPPORTED.
 *  TILE3D and STA keep copies of K (rotated with rope) and V in the workspace in
 *    tile-major order (2 x B*H*N_pad*d bf16), so that the attention loads each
 *    4x4x4 key tile as one run of 64 rows; q, k, v and out stay in raster order.
 *   out  bf16 [B][H][N_pad][d] device, written
 */
slr_status slr_frame_mask_attn(const void* q, const void* k, const void* v, const slr_seq* seq,
                               const slr_mask_desc* mask, void* out,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * slr_svoo_cocluster -- SVOO's online bidirectional co-clustering (gist.science
 * summary of SVOO, arXiv 2603.18636, section 3, stage 2).  Per (b, h): query
 * centres start at the anchor queries and key centres at the anchor keys; then
 * `iters` times
 *   step A: every valid key gets the label of the key centre whose affinity
 *           vector (its dot products with the query centres) is nearest in
 *           Euclidean distance to the key's own affinity vector (ties: the lower
 *           centre); each key centre moves to the mean of its keys (a centre
 *           with no key stays);
 *   step B: the same for every valid query against the key centres of step A,
 *           and the query centres move to their means.
 * Pad tokens get the label n_qc (queries) or n_kc (keys).  The permutations list
 * the tokens by ascending label, in token order within a label (a stable sort),
 * so that pads end them: they are the orders slr_svoo_attn takes.
 * Precision: the centres and their metric are formed in fp64 and kept in fp32;
 * the distances of the tokens to the centres come from the tensor cores with the
 * metric split into three bf16 terms (24 significant bits) and fp32
 * accumulation, so a label can differ from an exact evaluation only for a token
 * whose two nearest centres are within ~1e-6 (relative) of each other.  The call
 * is deterministic: the same inputs give the same outputs.
 *
 *   q, k        bf16 [B][H][N_pad][d] device, read only
 *   n_qc, n_kc  cluster counts, 2..128
 *   iters       iterations, >= 1 (the summary: about 2)
 *   q_anchor    int32 [B][H][n_qc] device: a valid query token per query centre
 *   k_anchor    int32 [B][H][n_kc] device: a valid key token per key centre
 *   q_label, k_label  int32 [B][H][N_pad] device, written
 *   q_perm, k_perm    int32 [B][H][N_pad] device, written: position -> token
 * Requires n_seg == 1 (one padded segment).  An anchor that is not a valid token
 * sets SLR_ERR_INDEX in the status word (its centre starts at 0).
 */
slr_status slr_svoo_cocluster(const void* q, const void* k, const slr_seq* seq, int n_qc, int n_kc, int iters,
                              const int32_t* q_anchor, const int32_t* k_anchor,
                              int32_t* q_label, int32_t* k_label, int32_t* q_perm, int32_t* k_perm,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * slr_svoo_attn -- softmax attention over the top block pairs of a co-clustered
 * order (SVOO summary, section 3, stage 2, block selection).  The rows of q are
 * taken in the order q_perm and those of k and v in the order k_perm; blocks are
 * 64 consecutive rows of those orders.  Within every query block the key blocks
 * are ranked by the SLA compressed score (as slr_pool_classify: block means,
 * softmax(pool(Q) pool(K)^T / sqrt(d)), ties to the lower index) and the top
 * kc = max(1, ceil(keep_frac * Nb)) are computed with exact softmax attention,
 * scale 1/sqrt(d); the others are skipped.  keep_frac = 1 computes every block
 * (the dense attention of the sequence, whatever the orders).  The output is
 * written back in the original token order.
 *
 *   q_perm, k_perm  int32 [B][H][N_pad] device: permutations of the tokens whose
 *                   first seg_len positions are the valid tokens (as
 *                   slr_svoo_cocluster writes them); an entry outside [0, N_pad)
 *                   sets SLR_ERR_INDEX; entries that repeat a token leave some
 *                   output rows unwritten
 *   keep_frac       in (0, 1]
 *   out             bf16 [B][H][N_pad][d] device, written (pad rows 0)
 *   mask_out_opt    int8 [B][H][Nb][Nb] device or NULL: 1 = computed pair, 0 =
 *                   skipped, over the blocks of the two orders
 * Requires n_seg == 1 and Nb <= 4096.  The workspace holds the reordered q, k, v
 * and output (4 x B*H*N_pad*d bf16).
 */
slr_status slr_svoo_attn(const void* q, const void* k, const void* v, const slr_seq* seq,
                         const int32_t* q_perm, const int32_t* k_perm, float keep_frac,
                         void* out, int8_t* mask_out_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * slr_block_sparse_attn_noalloc -- slr_block_sparse_attn without a workspace.
 * The source pages have no counterpart to this call; it exists for callers
 * that cannot allocate device memory for the library: a host application that
 * owns the whole device-memory budget (for example an inference server that
 * reserves the GPU's memory at start-up and forbids further cudaMalloc), or a
 * plug-in whose interface passes only input and output tensors.
 *
 * It computes exactly what slr_block_sparse_attn computes, with the same
 * arguments except `ws`/`ws_bytes`.  Its scratch (the status word, the
 * attention kernel's tile-queue counter and the per-pair key-block lists)
 * lives in one static device array of SLR_NOALLOC_SCRATCH_BYTES that every GPU
 * which loads the library holds until the process exits; the call allocates
 * nothing.
 *   status_opt  int device pointer or NULL: zeroed by the call, then receives
 *               the device status (0, or 5 / 6 for a timeout / an out-of-range
 *               index: the negated SLR_ERR_TIMEOUT / SLR_ERR_INDEX).  With NULL
 *               the status goes to the static array's status word (zeroed by
 *               the call as well), which slr_check_status(NULL, stream) reads.
 * Returns SLR_ERR_WORKSPACE when the lists of this shape need more than the
 * static scratch: 256 + B*H*ceil(Nb/2)*(min(Nb, 2*kv_max) + 1)*4 bytes (each
 * part rounded up to 256) must fit in SLR_NOALLOC_SCRATCH_BYTES; the dense mode
 * (kv_idx NULL) needs no lists.
 * The first call on each device looks up the device address of the static
 * array (cudaGetSymbolAddress, with that device current) and caches it; make
 * that first call before any stream capture.  All calls in the process share
 * the one array, which keeps the last call's lists: calls that can overlap on
 * the GPU (different streams, or different host threads on one device) race on
 * it -- on the lists, on the status word and, in every mode including the
 * dense one, on the tile-queue counter, so that an overlapping call can skip or
 * repeat tiles -- and must be serialised by the caller.
 */
#define SLR_NOALLOC_SCRATCH_BYTES (4u << 20)
slr_status slr_block_sparse_attn_noalloc(const void* q, const void* k, const void* v, const slr_seq* seq,
                                         const int32_t* kv_idx, const int32_t* kv_cnt, int kv_max,
                                         void* o, float* lse_opt, int* status_opt, void* stream);

/* ------------------------------------------------------------------ helpers */

/* Bytes of scratch the call `op` needs for this shape (0 on invalid input). */
size_t slr_workspace_bytes(int op, const slr_seq* seq, const void* params);

/* Synchronises `stream`, returns the status word that the device wrote into
 * `ws` since the last call started (SLR_OK if none), and clears it.  ws == NULL
 * reads (and clears) instead the status word of slr_block_sparse_attn_noalloc's
 * static scratch on the current device, where that call reports when it is
 * given no status pointer. */
slr_status slr_check_status(void* ws, void* stream);

/* Host-only: kc and kn for a row of n_kb key blocks (rule in slr_pool_classify). */
slr_status slr_block_counts(int n_kb, float crit_frac, float negl_frac, int* kc, int* kn);

/* Host-only: the LVSA attention sets A(t) for t = 0..T-1 at denoising step s
 * (rainbus page: T_per = ceil(T/(C-(2W+1))), G_s = {(s mod T_per + i*T_per) mod T},
 * adaptive window max(0, min(t-W, T-1-2W)) .. +2W, expanded toward the side
 * with more room -- a tie grows the right side -- until it holds
 * min(2W+1, T-|G|) non-global frames).  sets is host int32 [T][cap] with each
 * row ascending; counts is host int32 [T].  Requires C > 2W+1, T >= 1, and
 * cap >= the largest |A(t)| (SLR_ERR_ARG otherwise).  The device builds the
 * same sets with the same routine. */
slr_status slr_lvsa_attention_sets(int T, int C, int W, int step,
                                   int32_t* sets, int32_t* counts, int cap);

/* Per-kernel timing (host side).  slr_profile_enable(1) makes every later
 * launch of this process record a CUDA event pair on the launch's own stream
 * (event objects are created on first use and reused; this is the one place
 * the library creates CUDA resources).  slr_profile_collect() synchronises
 * those events, writes for up to `max` kernel kinds their name, launch count
 * and total device milliseconds since the last collect, clears the record,
 * and returns the number of kinds written.  slr_profile_enable(0) stops
 * recording.  Not thread-safe: profile from one host thread. */
slr_status slr_profile_enable(int on);
int slr_profile_collect(const char** names, int* launches, double* total_ms, int max);

const char* slr_status_string(slr_status s);
/* ABI version, 100 * major + minor.  200: slr_mask_desc gained `rope` and `window` (and the
 * SLR_MASK_STA kind), so a caller built against an earlier header passes a shorter struct.
 * 201: the SVOO calls slr_svoo_cocluster and slr_svoo_attn. */
#define SLR_ABI_VERSION 201
int slr_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SLR_H */
