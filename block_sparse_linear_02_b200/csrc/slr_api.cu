// slr_api.cu -- the C ABI of libslr (declared in include/slr.h): argument
// validation, workspace layout, and the launch sequence of every entry point.
// Nothing here synchronises or allocates (except slr_check_status, which is
// documented to synchronise).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/slr.h"
#include "launch.h"
#include "lvsa_sets.cuh"

namespace slr {

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tile_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    default: return false;
  }
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) { gdim[i] = dims[i]; bdim[i] = box[i]; estr[i] = 1; }
  for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), gdim, gstr,
                  bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace slr

using namespace slr;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Sequential carving of the caller's workspace.  With base == nullptr it only counts.
struct Carve {
  uint8_t* base;
  size_t off;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)), off(0) {}
  template <class T>
  T* take(size_t count) {
    const size_t at = off;
    off = align_up(off + count * sizeof(T));
    return base ? reinterpret_cast<T*>(base + at) : nullptr;
  }
};

struct Shape {
  int B, H, BH, d, n_seg, seg_len, seg_stride, n_pad, nb, npairs;
  SeqShape s;
};

slr_status check_seq(const slr_seq* q, Shape& sh) {
  if (!q) return SLR_ERR_ARG;
  if (q->B < 1 || q->H < 1 || q->n_seg < 1 || q->seg_len < 1 || q->seg_stride < 1) return SLR_ERR_ARG;
  if (q->d != 64 && q->d != 128) return SLR_ERR_UNSUPPORTED;
  if (q->block != kBlock) return SLR_ERR_UNSUPPORTED;
  if (q->seg_stride % kBlock != 0) return SLR_ERR_UNSUPPORTED;
  if (q->seg_len > q->seg_stride || q->seg_len <= q->seg_stride - kBlock) return SLR_ERR_UNSUPPORTED;
  const long long n_pad = (long long)q->n_seg * q->seg_stride;
  if (n_pad / kBlock > kMaxKeyBlocks) return SLR_ERR_UNSUPPORTED;
  const long long bh = (long long)q->B * q->H;
  if (bh > 65535) return SLR_ERR_UNSUPPORTED;
  sh.B = q->B; sh.H = q->H; sh.BH = (int)bh; sh.d = q->d;
  sh.n_seg = q->n_seg; sh.seg_len = q->seg_len; sh.seg_stride = q->seg_stride;
  sh.n_pad = (int)n_pad; sh.nb = (int)(n_pad / kBlock); sh.npairs = (sh.nb + 1) / 2;
  sh.s = SeqShape{sh.n_pad, sh.seg_len, sh.seg_stride, sh.nb};
  return SLR_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

slr_status counts(int nb, float crit, float negl, int* kc, int* kn) {
  if (!(crit >= 0.f && crit <= 1.f && negl >= 0.f && negl <= 1.f)) return SLR_ERR_ARG;
  if ((double)crit + (double)negl > 1.0 + 1e-6) return SLR_ERR_ARG;
  const double c = (double)crit * nb, n = (double)negl * nb;
  int a = (int)ceil(c - 1e-3);
  if (a < 1) a = 1;
  if (a > nb) a = nb;
  int b = (int)floor(n + 1e-3);
  if (b < 0) b = 0;
  if (b > nb - a) b = nb - a;
  *kc = a;
  *kn = b;
  return SLR_OK;
}

int ld_m01(int nb) { return (nb + 63) / 64 * 64; }

// ---------------------------------------------------------------- workspace plans

struct ClassifyWs {
  __nv_bfloat16 *qsplit, *ksplit;
  uint32_t* keys;
  __nv_bfloat16* m01;
  __nv_bfloat16* phi_q;                // phi(q) for the linear branch (SLA with marginal blocks)
};

void plan_classify(Carve& c, const Shape& sh, bool m01, ClassifyWs& w) {
  w.qsplit = c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * 3 * sh.d);
  w.ksplit = c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * 3 * sh.d);
  w.keys = c.take<uint32_t>((size_t)sh.BH * sh.nb * logits_row_stride(sh.nb));
  w.m01 = m01 ? c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * ld_m01(sh.nb)) : nullptr;
  w.phi_q = m01 ? c.take<__nv_bfloat16>((size_t)sh.BH * sh.s.n_pad * sh.d) : nullptr;
}

struct MarginalWs {
  __nv_bfloat16 *h, *Hs;
};

void plan_marginal(Carve& c, const Shape& sh, MarginalWs& w) {
  const size_t per = (size_t)(sh.d + 1) * sh.d;
  w.h = c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * per);
  w.Hs = c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * per);
}

struct SlaWs {
  int* status;
  ClassifyWs cls;
  uint32_t* list;
  int32_t* list_cnt;
  int cap;
  MarginalWs mar;
};

void plan_sla(Carve& c, const Shape& sh, int kc, int kn, SlaWs& w) {
  w.status = c.take<int>(64);
  const bool dense = kc == sh.nb;
  w.cap = dense ? 0 : (2 * kc < sh.nb ? 2 * kc : sh.nb);
  if (dense) return;
  plan_classify(c, sh, sh.nb - kc - kn > 0, w.cls);
  w.list = c.take<uint32_t>((size_t)sh.BH * sh.npairs * w.cap);
  w.list_cnt = c.take<int32_t>((size_t)sh.BH * sh.npairs);
  if (sh.nb - kc - kn > 0) {
    plan_marginal(c, sh, w.mar);
  } else {
    w.mar.h = w.mar.Hs = nullptr;
  }
}

struct FrameWs {
  int* status;
  int32_t *sets, *set_cnt;
  int set_cap;
  uint32_t* list;
  int32_t* list_cnt;
  int cap;
  void *kf, *vf;
  void* qr;          // rotated q, raster order (TILE3D with rope)
  void *kt, *vt;     // K (rotated with rope) and V in tile-major order (TILE3D, STA)
  void *tab, *part;  // TILE3D: RoPE cos / sin table, far-field row sums
};

slr_status check_mask(const slr_mask_desc* m, const Shape& sh) {
  if (!m) return SLR_ERR_ARG;
  if (m->kind == SLR_MASK_LVSA) {
    if (m->T != sh.n_seg || m->W < 0 || m->step < 0 || m->C <= 2 * m->W + 1) return SLR_ERR_ARG;
    if (m->rope != 0) return SLR_ERR_UNSUPPORTED;
    return SLR_OK;
  }
  if (m->kind == SLR_MASK_TILE3D) {
    if (sh.n_seg != 1 || sh.seg_len != sh.seg_stride) return SLR_ERR_UNSUPPORTED;
    if (m->F < 1 || m->Hh < 1 || m->Ww < 1) return SLR_ERR_ARG;
    if ((long long)m->F * m->Hh * m->Ww != sh.n_pad) return SLR_ERR_ARG;
    if (m->tile[0] != 4 || m->tile[1] != 4 || m->tile[2] != 4) return SLR_ERR_UNSUPPORTED;
    if (m->F % 4 || m->Hh % 4 || m->Ww % 4) return SLR_ERR_UNSUPPORTED;
    if (m->radius < 0) return SLR_ERR_ARG;
    const int* c = m->cell;
    if (c[0] < 1 || c[1] < 1 || c[2] < 1 || m->F % c[0] || m->Hh % c[1] || m->Ww % c[2]) return SLR_ERR_ARG;
    if ((m->F / c[0]) * (m->Hh / c[1]) * (m->Ww / c[2]) != 64) return SLR_ERR_UNSUPPORTED;
    if (!(m->gate >= 0.f && m->gate <= 1.f)) return SLR_ERR_ARG;
    if (m->rope != 0 && m->rope != 1) return SLR_ERR_ARG;
    if ((size_t)m->Ww * sh.d * 2 > kFarRowBytesMax) return SLR_ERR_UNSUPPORTED;
    return SLR_OK;
  }
  if (m->kind == SLR_MASK_STA) {
    if (sh.n_seg != 1 || sh.seg_len != sh.seg_stride) return SLR_ERR_UNSUPPORTED;
    if (m->F < 1 || m->Hh < 1 || m->Ww < 1) return SLR_ERR_ARG;
    if ((long long)m->F * m->Hh * m->Ww != sh.n_pad) return SLR_ERR_ARG;
    if (m->tile[0] != 4 || m->tile[1] != 4 || m->tile[2] != 4) return SLR_ERR_UNSUPPORTED;
    if (m->F % 4 || m->Hh % 4 || m->Ww % 4) return SLR_ERR_UNSUPPORTED;
    for (int a = 0; a < 3; ++a)            // an odd number of whole tiles
      if (m->window[a] < 4 || m->window[a] % 4 || (m->window[a] / 4) % 2 == 0) return SLR_ERR_ARG;
    if (m->rope != 0) return SLR_ERR_UNSUPPORTED;
    return SLR_OK;
  }
  return SLR_ERR_ARG;
}

// Tile radius per axis of a TILE3D or STA mask: a window of (2r+1) tiles keeps the tiles
// whose centres lie within half a window of the query tile's centre, i.e. within r tiles
// A radius past the grid adds no tile, so it is clamped to the grid's extent on that axis.
void mask_radii(const slr_mask_desc* m, int rad[3]) {
  const int extent[3] = {m->F / 4, m->Hh / 4, m->Ww / 4};
  for (int a = 0; a < 3; ++a) {
    const int r = m->kind == SLR_MASK_STA ? (m->window[a] / 4 - 1) / 2 : m->radius;
    rad[a] = r < extent[a] - 1 ? r : extent[a] - 1;
  }
}

void plan_frame(Carve& c, const Shape& sh, const slr_mask_desc* m, FrameWs& w) {
  w.status = c.take<int>(64);
  w.sets = w.set_cnt = nullptr;
  w.kf = w.vf = nullptr;
  w.qr = w.kt = w.vt = w.tab = w.part = nullptr;
  if (m->kind == SLR_MASK_LVSA) {
    const LvsaGlobals g = lvsa_globals(m->T, m->C, m->W, m->step);
    const int win = (2 * m->W + 1 < m->T - g.count) ? 2 * m->W + 1 : m->T - g.count;
    w.set_cap = g.count + win;
    w.sets = c.take<int32_t>((size_t)m->T * w.set_cap);
    w.set_cnt = c.take<int32_t>((size_t)m->T);
    const int bpf = sh.seg_stride / kBlock;
    const long long cap = 2LL * w.set_cap * bpf;
    w.cap = cap < sh.nb ? (int)cap : sh.nb;
  } else {
    int rad[3];
    mask_radii(m, rad);
    const long long cap = 2LL * (2 * rad[0] + 1) * (2 * rad[1] + 1) * (2 * rad[2] + 1);
    w.cap = cap < sh.nb ? (int)cap : sh.nb;
    w.set_cap = 0;
    if (m->kind == SLR_MASK_TILE3D) {
      w.kf = c.take<__nv_bfloat16>((size_t)sh.BH * 64 * sh.d);
      w.vf = c.take<__nv_bfloat16>((size_t)sh.BH * 64 * sh.d);
      w.part = c.take<uint8_t>(far_partial_bytes(sh.BH, sh.d, m->F, m->Hh, m->Ww, m->cell[2]));
      if (m->rope) w.tab = c.take<uint8_t>(far_rope_table_bytes(sh.d, m->F, m->Hh, m->Ww));
    }
    w.kt = c.take<__nv_bfloat16>((size_t)sh.BH * sh.n_pad * sh.d);
    w.vt = c.take<__nv_bfloat16>((size_t)sh.BH * sh.n_pad * sh.d);
    if (m->rope) w.qr = c.take<__nv_bfloat16>((size_t)sh.BH * sh.n_pad * sh.d);
  }
  w.list = c.take<uint32_t>((size_t)sh.npairs * w.cap);
  w.list_cnt = c.take<int32_t>((size_t)sh.npairs);
}

struct SvooClusterWs {
  int* status;
  float *cq, *ck;                      // centres [BH][Cp][d]
  __nv_bfloat16* ub;                   // metric of the assigning side [BH][Cp][3d]
  float* bias;                         // [BH][Cp]
  int32_t *counts, *offs, *start;      // counting sort
  int32_t* poff;                       // piece offsets of the centre update
  double* part;                        // fp64 piece sums of the centre update
};

void plan_svoo_cluster(Carve& c, const Shape& sh, int n_qc, int n_kc, SvooClusterWs& w) {
  const int cpq = svoo_padded_clusters(n_qc), cpk = svoo_padded_clusters(n_kc);
  const int cpm = cpq > cpk ? cpq : cpk, cm = n_qc > n_kc ? n_qc : n_kc;
  const size_t nch = (size_t)svoo_sort_chunks(sh.n_pad);
  w.status = c.take<int>(64);
  w.cq = c.take<float>((size_t)sh.BH * cpq * sh.d);
  w.ck = c.take<float>((size_t)sh.BH * cpk * sh.d);
  w.ub = c.take<__nv_bfloat16>((size_t)sh.BH * cpm * 3 * sh.d);
  w.bias = c.take<float>((size_t)sh.BH * cpm);
  w.counts = c.take<int32_t>((size_t)sh.BH * nch * (cm + 1));
  w.offs = c.take<int32_t>((size_t)sh.BH * nch * (cm + 1));
  w.start = c.take<int32_t>((size_t)sh.BH * (cm + 2));
  w.poff = c.take<int32_t>((size_t)sh.BH * (cm + 1));
  w.part = c.take<double>((size_t)sh.BH * svoo_max_pieces(sh.n_pad, cm) * sh.d);
}

struct SvooAttnWs {
  int* status;
  ClassifyWs cls;
  uint32_t* list;
  int32_t* list_cnt;
  int cap;
  void *qp, *kp, *vp, *op;             // the reordered q, k, v and the output in that order
};

void plan_svoo_attn(Carve& c, const Shape& sh, int kc, SvooAttnWs& w) {
  w.status = c.take<int>(64);
  const bool dense = kc == sh.nb;
  w.cap = dense ? 0 : (2 * kc < sh.nb ? 2 * kc : sh.nb);
  if (!dense) {
    plan_classify(c, sh, false, w.cls);
    w.list = c.take<uint32_t>((size_t)sh.BH * sh.npairs * w.cap);
    w.list_cnt = c.take<int32_t>((size_t)sh.BH * sh.npairs);
  } else {
    w.list = nullptr;
    w.list_cnt = nullptr;
  }
  const size_t rows = (size_t)sh.BH * sh.n_pad * sh.d;
  w.qp = c.take<__nv_bfloat16>(rows);
  w.kp = c.take<__nv_bfloat16>(rows);
  w.vp = c.take<__nv_bfloat16>(rows);
  w.op = c.take<__nv_bfloat16>(rows);
}

slr_status ws_check(void* ws, size_t have, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return SLR_ERR_WORKSPACE;
  if (have < need) return SLR_ERR_WORKSPACE;
  return SLR_OK;
}

#define SLR_TRY(expr)                                   \
  do {                                                  \
    if ((expr) != cudaSuccess) return SLR_ERR_CUDA;     \
  } while (0)

// ---------------------------------------------------------------- per-kernel profiler
enum KernelKind {
  kKPool, kKLogits, kKClassify, kKLists, kKKeyStates, kKReduce, kKApply, kKAttention, kKLvsaSets,
  kKFarPool, kKMaskToM01, kKTileMajor, kKSvooAnchors, kKSvooAssign, kKSvooSort, kKSvooUpdate, kKSvooGather,
  kKSvooScatter, kKNumKinds
};
const char* const kKindNames[kKNumKinds] = {
    "pool_means", "logits", "classify", "pair_lists", "key_states", "reduce_states",
    "linear_apply", "attention", "lvsa_sets", "far_pool", "mask_to_m01", "tile_major",
    "svoo_anchors", "svoo_assign", "svoo_sort", "svoo_update", "svoo_gather", "svoo_scatter"};

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
bool g_prof = false;
cudaEvent_t g_pool[4096];
int g_pool_n = 0;
ProfRec g_pending[2048];
int g_pending_n = 0;
int g_launches[kKNumKinds];
double g_ms[kKNumKinds];

cudaEvent_t prof_event() {
  if (g_pool_n > 0) return g_pool[--g_pool_n];
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void prof_drain() {
  for (int i = 0; i < g_pending_n; ++i) {
    ProfRec& r = g_pending[i];
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      g_launches[r.kind] += 1;
      g_ms[r.kind] += ms;
    }
    if (g_pool_n + 2 <= 4096) { g_pool[g_pool_n++] = r.a; g_pool[g_pool_n++] = r.b; }
  }
  g_pending_n = 0;
}

struct ProfScope {
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  ProfScope(int k, cudaStream_t s) : kind(k), st(s) {
    if (g_prof) {
      if (g_pending_n >= 2048) prof_drain();
      a = prof_event();
      cudaEventRecord(a, st);
    }
  }
  ~ProfScope() {
    if (a) {
      cudaEvent_t b = prof_event();
      cudaEventRecord(b, st);
      g_pending[g_pending_n++] = ProfRec{kind, a, b};
    }
  }
};

// Launch `expr` (a launcher call) bracketed by profiler events when profiling is on.
#define SLR_LAUNCH(kind, stream, expr)                  \
  do {                                                  \
    ProfScope _ps(kind, stream);                        \
    if ((expr) != cudaSuccess) return SLR_ERR_CUDA;     \
  } while (0)

AttnArgs attn_base(const Shape& sh, const void* q, const void* k, const void* v, void* out, int* status) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v;
  a.BH = sh.BH; a.d = sh.d; a.s = sh.s;
  a.n_qb = sh.nb; a.n_kb = sh.nb; a.n_pairs = sh.npairs;
  a.out = out;
  a.status = status;
  a.tile_counter = status + 1;   // the status area holds 64 ints
  a.gate = 1.f;
  return a;
}

}  // namespace

extern "C" {

int slr_version(void) { return SLR_ABI_VERSION; }

slr_status slr_profile_enable(int on) {
  g_prof = on != 0;
  return SLR_OK;
}

int slr_profile_collect(const char** names, int* launches, double* total_ms, int max) {
  prof_drain();
  int n = 0;
  for (int k = 0; k < kKNumKinds; ++k) {
    if (g_launches[k] == 0) continue;
    if (n < max) {
      if (names) names[n] = kKindNames[k];
      if (launches) launches[n] = g_launches[k];
      if (total_ms) total_ms[n] = g_ms[k];
      ++n;
    }
    g_launches[k] = 0;
    g_ms[k] = 0.0;
  }
  return n;
}

const char* slr_status_string(slr_status s) {
  switch (s) {
    case SLR_OK: return "ok";
    case SLR_ERR_ARG: return "invalid argument";
    case SLR_ERR_UNSUPPORTED: return "unsupported shape";
    case SLR_ERR_WORKSPACE: return "workspace too small or misaligned";
    case SLR_ERR_CUDA: return "CUDA error";
    case SLR_ERR_TIMEOUT: return "device wait timed out";
    case SLR_ERR_INDEX: return "block index out of range";
    default: return "unknown status";
  }
}

slr_status slr_block_counts(int n_kb, float crit_frac, float negl_frac, int* kc, int* kn) {
  if (n_kb < 1 || !kc || !kn) return SLR_ERR_ARG;
  return counts(n_kb, crit_frac, negl_frac, kc, kn);
}

slr_status slr_lvsa_attention_sets(int T, int C, int W, int step, int32_t* sets, int32_t* cnts, int cap) {
  if (T < 1 || W < 0 || step < 0 || C <= 2 * W + 1 || !sets || !cnts || cap < 1) return SLR_ERR_ARG;
  for (int t = 0; t < T; ++t) {
    const int n = lvsa_attention_set(T, C, W, step, t, sets + (size_t)t * cap, cap);
    if (n < 0) return SLR_ERR_ARG;
    cnts[t] = n;
  }
  return SLR_OK;
}

size_t slr_workspace_bytes(int op, const slr_seq* seq, const void* params) {
  Shape sh;
  if (check_seq(seq, sh) != SLR_OK) return 0;
  Carve c(nullptr);
  switch (op) {
    case SLR_OP_POOL_CLASSIFY: {
      if (sh.nb > kMaxClassifyBlocks || !params) return 0;
      c.take<int>(64);
      ClassifyWs w;
      plan_classify(c, sh, false, w);
      return c.off;
    }
    case SLR_OP_BLOCK_SPARSE: {
      c.take<int>(64);
      const int kv_max = params ? *static_cast<const int*>(params) : sh.nb;
      const int cap = (int)(2LL * kv_max < sh.nb ? 2LL * kv_max : sh.nb);
      c.take<uint32_t>((size_t)sh.BH * sh.npairs * (cap > 0 ? cap : 1));
      c.take<int32_t>((size_t)sh.BH * sh.npairs);
      return c.off;
    }
    case SLR_OP_LINEAR_MARGINAL: {
      c.take<int>(64);
      c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * ld_m01(sh.nb));
      MarginalWs w;
      plan_marginal(c, sh, w);
      return c.off;
    }
    case SLR_OP_SPARSE_LINEAR: {
      if (!params) return 0;
      const slr_fracs* f = static_cast<const slr_fracs*>(params);
      int kc, kn;
      if (counts(sh.nb, f->crit_frac, f->negl_frac, &kc, &kn) != SLR_OK) return 0;
      if (kc != sh.nb && sh.nb > kMaxClassifyBlocks) return 0;
      SlaWs w;
      plan_sla(c, sh, kc, kn, w);
      return c.off;
    }
    case SLR_OP_FRAME_MASK: {
      const slr_mask_desc* m = static_cast<const slr_mask_desc*>(params);
      if (check_mask(m, sh) != SLR_OK) return 0;
      FrameWs w;
      plan_frame(c, sh, m, w);
      return c.off;
    }
    case SLR_OP_SVOO_COCLUSTER: {
      const int* cl = static_cast<const int*>(params);
      if (!cl || sh.n_seg != 1) return 0;
      if (cl[0] < 2 || cl[0] > kSvooMaxClusters || cl[1] < 2 || cl[1] > kSvooMaxClusters) return 0;
      SvooClusterWs w;
      plan_svoo_cluster(c, sh, cl[0], cl[1], w);
      return c.off;
    }
    case SLR_OP_SVOO_ATTN: {
      const float* keep = static_cast<const float*>(params);
      if (!keep || sh.n_seg != 1) return 0;
      int kc, kn;
      if (!(*keep > 0.f) || counts(sh.nb, *keep, 0.f, &kc, &kn) != SLR_OK) return 0;
      if (kc != sh.nb && sh.nb > kMaxClassifyBlocks) return 0;
      SvooAttnWs w;
      plan_svoo_attn(c, sh, kc, w);
      return c.off;
    }
    default:
      return 0;
  }
}

slr_status slr_check_status(void* ws, void* stream) {
  if (!ws) return noalloc_check_status(stream);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SLR_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SLR_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return SLR_ERR_CUDA;
  return code == 0 ? SLR_OK : -code;
}

slr_status slr_pool_classify(const void* q, const void* k, const slr_seq* seq, float crit_frac, float negl_frac,
                             int8_t* mask, int32_t* crit_idx, int32_t* crit_cnt, float* scores_opt,
                             void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (sh.nb > kMaxClassifyBlocks) return SLR_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !mask || !crit_idx || !crit_cnt) return SLR_ERR_ARG;
  int kc, kn;
  if ((st = counts(sh.nb, crit_frac, negl_frac, &kc, &kn)) != SLR_OK) return st;
  const slr_fracs f{crit_frac, negl_frac};
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_POOL_CLASSIFY, seq, &f))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  int* status = c.take<int>(64);
  ClassifyWs w;
  plan_classify(c, sh, false, w);
  SLR_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  SLR_LAUNCH(kKPool, s, launch_pool_means(q, k, w.qsplit, w.ksplit, nullptr, SLR_PHI_ELU1, sh.BH, sh.d, sh.s, s));
  SLR_LAUNCH(kKLogits, s, launch_logits(w.qsplit, w.ksplit, w.keys, sh.BH, sh.nb, sh.d, status, s));
  SLR_LAUNCH(kKClassify, s, launch_classify(w.keys, sh.BH, sh.nb, sh.d, kc, kn, mask, crit_idx, crit_cnt,
                                            nullptr, 0, scores_opt, nullptr, nullptr, 0, sh.s, status, s));
  return SLR_OK;
}

slr_status slr_block_sparse_attn(const void* q, const void* k, const void* v, const slr_seq* seq,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, int kv_max,
                                 void* o, float* lse_opt, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SLR_ERR_ARG;
  if (kv_idx && (!kv_cnt || kv_max < 1)) return SLR_ERR_ARG;
  const int km = kv_idx ? kv_max : sh.nb;
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_BLOCK_SPARSE, seq, &km))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  int* status = c.take<int>(64);
  const int cap = (int)(2LL * km < sh.nb ? 2LL * km : sh.nb);
  uint32_t* list = c.take<uint32_t>((size_t)sh.BH * sh.npairs * cap);
  int32_t* list_cnt = c.take<int32_t>((size_t)sh.BH * sh.npairs);
  SLR_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  AttnArgs a = attn_base(sh, q, k, v, o, status);
  a.lse = lse_opt;
  if (kv_idx) {
    ListArgs la;
    memset(&la, 0, sizeof(la));
    la.mode = kListExplicit;
    la.n_qb = sh.nb; la.n_kb = sh.nb; la.n_pairs = sh.npairs; la.cap = cap;
    la.kv_idx = kv_idx; la.kv_cnt = kv_cnt; la.kv_max = kv_max;
    la.s = sh.s; la.list = list; la.list_cnt = list_cnt; la.status = status;
    SLR_LAUNCH(kKLists, s, launch_pair_lists(la, sh.BH, s));
    a.list = list; a.list_cnt = list_cnt; a.list_cap = cap; a.list_per_head = 1;
  }
  SLR_LAUNCH(kKAttention, s, launch_attention(a, s));
  return SLR_OK;
}

slr_status slr_linear_marginal(const void* q, const void* k, const void* v, const slr_seq* seq,
                               const int8_t* mask, int phi, const void* w_proj_opt,
                               float* o_lin, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !mask || !aligned16(o_lin)) return SLR_ERR_ARG;
  if (w_proj_opt && !aligned16(w_proj_opt)) return SLR_ERR_ARG;
  if (phi != SLR_PHI_ELU1 && phi != SLR_PHI_SOFTMAX) return SLR_ERR_UNSUPPORTED;
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_LINEAR_MARGINAL, seq, nullptr))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  int* status = c.take<int>(64);
  __nv_bfloat16* m01 = c.take<__nv_bfloat16>((size_t)sh.BH * sh.nb * ld_m01(sh.nb));
  MarginalWs w;
  plan_marginal(c, sh, w);
  SLR_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  SLR_LAUNCH(kKMaskToM01, s, launch_mask_to_m01(mask, m01, sh.BH, sh.nb, ld_m01(sh.nb), s));
  SLR_LAUNCH(kKKeyStates, s, launch_key_states(k, v, w_proj_opt, w.h, phi, sh.BH, sh.d, sh.s, status, s));
  SLR_LAUNCH(kKReduce, s, launch_reduce_states(m01, ld_m01(sh.nb), w.h, w.Hs, sh.BH, sh.nb, sh.d, status, s));
  SLR_LAUNCH(kKApply, s, launch_linear_apply(q, w.Hs, o_lin, phi, sh.BH, sh.d, sh.s, status, s));
  return SLR_OK;
}

slr_status slr_sparse_linear_attn(const void* q, const void* k, const void* v, const void* w_proj,
                                  const slr_seq* seq, float crit_frac, float negl_frac, int phi,
                                  void* out, int8_t* mask_out_opt, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SLR_ERR_ARG;
  if (phi != SLR_PHI_ELU1 && phi != SLR_PHI_SOFTMAX) return SLR_ERR_UNSUPPORTED;
  int kc, kn;
  if ((st = counts(sh.nb, crit_frac, negl_frac, &kc, &kn)) != SLR_OK) return st;
  const bool dense = kc == sh.nb;
  const bool marginal = !dense && sh.nb - kc - kn > 0;
  if (marginal && !aligned16(w_proj)) return SLR_ERR_ARG;
  if (!dense && sh.nb > kMaxClassifyBlocks) return SLR_ERR_UNSUPPORTED;
  const slr_fracs f{crit_frac, negl_frac};
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_SPARSE_LINEAR, seq, &f))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  SlaWs w;
  plan_sla(c, sh, kc, kn, w);
  SLR_TRY(cudaMemsetAsync(w.status, 0, sizeof(int), s));
  AttnArgs a = attn_base(sh, q, k, v, out, w.status);
  if (dense) {
    if (mask_out_opt) SLR_TRY(cudaMemsetAsync(mask_out_opt, 1, (size_t)sh.BH * sh.nb * sh.nb, s));
    SLR_LAUNCH(kKAttention, s, launch_attention(a, s));
    return SLR_OK;
  }
  SLR_LAUNCH(kKPool, s, launch_pool_means(q, k, w.cls.qsplit, w.cls.ksplit, w.cls.phi_q, phi, sh.BH, sh.d, sh.s, s));
  SLR_LAUNCH(kKLogits, s, launch_logits(w.cls.qsplit, w.cls.ksplit, w.cls.keys, sh.BH, sh.nb, sh.d, w.status, s));
  SLR_LAUNCH(kKClassify, s, launch_classify(w.cls.keys, sh.BH, sh.nb, sh.d, kc, kn, mask_out_opt, nullptr,
                                            nullptr, w.cls.m01, ld_m01(sh.nb), nullptr, w.list, w.list_cnt, w.cap,
                                            sh.s, w.status, s));
  if (marginal) {
    SLR_LAUNCH(kKKeyStates, s, launch_key_states(k, v, w_proj, w.mar.h, phi, sh.BH, sh.d, sh.s, w.status, s));
    SLR_LAUNCH(kKReduce, s, launch_reduce_states(w.cls.m01, ld_m01(sh.nb), w.mar.h, w.mar.Hs, sh.BH, sh.nb, sh.d, w.status, s));
    a.Hs = w.mar.Hs;
    a.phi_q = w.cls.phi_q;
  }
  a.list = w.list; a.list_cnt = w.list_cnt; a.list_cap = w.cap; a.list_per_head = 1;
  SLR_LAUNCH(kKAttention, s, launch_attention(a, s));
  return SLR_OK;
}

slr_status slr_frame_mask_attn(const void* q, const void* k, const void* v, const slr_seq* seq,
                               const slr_mask_desc* m, void* out, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SLR_ERR_ARG;
  if ((st = check_mask(m, sh)) != SLR_OK) return st;
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_FRAME_MASK, seq, m))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  FrameWs w;
  plan_frame(c, sh, m, w);
  SLR_TRY(cudaMemsetAsync(w.status, 0, sizeof(int), s));
  ListArgs la;
  memset(&la, 0, sizeof(la));
  la.n_qb = sh.nb; la.n_kb = sh.nb; la.n_pairs = sh.npairs; la.cap = w.cap;
  la.s = sh.s; la.list = w.list; la.list_cnt = w.list_cnt; la.status = w.status;
  AttnArgs a = attn_base(sh, q, k, v, out, w.status);
  if (m->kind == SLR_MASK_LVSA) {
    SLR_LAUNCH(kKLvsaSets, s, launch_lvsa_sets(m->T, m->C, m->W, m->step, w.sets, w.set_cnt, w.set_cap, s));
    la.mode = kListLvsa;
    la.sets = w.sets; la.set_cnt = w.set_cnt; la.set_cap = w.set_cap;
    la.blocks_per_frame = sh.seg_stride / kBlock;
  } else {
    la.mode = kListTile3d;
    la.TF = m->F / 4; la.TH = m->Hh / 4; la.TW = m->Ww / 4;
    mask_radii(m, la.rad);
    a.tile3d = 1; a.F = m->F; a.Hh = m->Hh; a.Ww = m->Ww;
    // the attention loads every key tile as 64 consecutive rows of tile-major K and V
    a.k = w.kt;
    a.v = w.vt;
  }
  if (m->kind == SLR_MASK_STA) {
    SLR_LAUNCH(kKTileMajor, s, launch_tile_major(k, v, w.kt, w.vt, sh.BH, sh.d, m->F, m->Hh, m->Ww, s));
  } else if (m->kind == SLR_MASK_TILE3D) {
    // the pooling pass writes tile-major K and V, and with the rotary embedding it also
    // rotates q and k (once, for both branches: the far field pools the rotated K)
    SLR_LAUNCH(kKFarPool, s, launch_far_field(q, k, v, w.qr, w.kt, w.vt, w.kf, w.vf, w.tab, w.part, sh.BH, sh.d,
                                              m->F, m->Hh, m->Ww, m->cell[0], m->cell[1], m->cell[2], m->rope, s));
    if (m->rope) a.q = w.qr;
    a.gated = 1; a.gate = m->gate; a.kf = w.kf; a.vf = w.vf;
  }
  SLR_LAUNCH(kKLists, s, launch_pair_lists(la, 1, s));
  a.list = w.list; a.list_cnt = w.list_cnt; a.list_cap = w.cap; a.list_per_head = 0;
  SLR_LAUNCH(kKAttention, s, launch_attention(a, s));
  return SLR_OK;
}

slr_status slr_svoo_cocluster(const void* q, const void* k, const slr_seq* seq, int n_qc, int n_kc, int iters,
                              const int32_t* q_anchor, const int32_t* k_anchor, int32_t* q_label, int32_t* k_label,
                              int32_t* q_perm, int32_t* k_perm, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (sh.n_seg != 1) return SLR_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !q_anchor || !k_anchor || !q_label || !k_label || !q_perm || !k_perm)
    return SLR_ERR_ARG;
  if (n_qc < 2 || n_qc > kSvooMaxClusters || n_kc < 2 || n_kc > kSvooMaxClusters || iters < 1) return SLR_ERR_ARG;
  const int cl[2] = {n_qc, n_kc};
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_SVOO_COCLUSTER, seq, cl))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  SvooClusterWs w;
  plan_svoo_cluster(c, sh, n_qc, n_kc, w);
  const int cm = n_qc > n_kc ? n_qc : n_kc;
  SLR_TRY(cudaMemsetAsync(w.status, 0, sizeof(int), s));
  SLR_TRY(cudaMemsetAsync(w.counts, 0, (size_t)sh.BH * svoo_sort_chunks(sh.n_pad) * (cm + 1) * sizeof(int32_t), s));
  SLR_LAUNCH(kKSvooAnchors, s, launch_svoo_anchors(q, q_anchor, w.cq, n_qc, sh.BH, sh.d, sh.s, w.status, s));
  SLR_LAUNCH(kKSvooAnchors, s, launch_svoo_anchors(k, k_anchor, w.ck, n_kc, sh.BH, sh.d, sh.s, w.status, s));
  for (int it = 0; it < iters; ++it) {
    // step A: the keys against the query centres, then the key centres move
    SLR_LAUNCH(kKSvooAssign, s, launch_svoo_assign(k, w.cq, n_qc, w.ck, n_kc, w.ub, w.bias, k_label, w.counts,
                                                   sh.BH, sh.d, sh.s, w.status, s));
    SLR_LAUNCH(kKSvooSort, s, launch_svoo_sort(k_label, w.counts, w.offs, w.start, w.poff, k_perm, n_kc, sh.BH,
                                               sh.s, s));
    SLR_LAUNCH(kKSvooUpdate, s, launch_svoo_update(k, k_perm, w.start, w.poff, w.part, w.ck, n_kc, sh.BH, sh.d,
                                                   sh.s, s));
    // step B: the queries against the updated key centres
    SLR_LAUNCH(kKSvooAssign, s, launch_svoo_assign(q, w.ck, n_kc, w.cq, n_qc, w.ub, w.bias, q_label, w.counts,
                                                   sh.BH, sh.d, sh.s, w.status, s));
    SLR_LAUNCH(kKSvooSort, s, launch_svoo_sort(q_label, w.counts, w.offs, w.start, w.poff, q_perm, n_qc, sh.BH,
                                               sh.s, s));
    if (it + 1 < iters)
      SLR_LAUNCH(kKSvooUpdate, s, launch_svoo_update(q, q_perm, w.start, w.poff, w.part, w.cq, n_qc, sh.BH, sh.d,
                                                     sh.s, s));
  }
  return SLR_OK;
}

slr_status slr_svoo_attn(const void* q, const void* k, const void* v, const slr_seq* seq, const int32_t* q_perm,
                         const int32_t* k_perm, float keep_frac, void* out, int8_t* mask_out_opt, void* ws,
                         size_t ws_bytes, void* stream) {
  Shape sh;
  slr_status st = check_seq(seq, sh);
  if (st != SLR_OK) return st;
  if (sh.n_seg != 1) return SLR_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !q_perm || !k_perm) return SLR_ERR_ARG;
  if (!(keep_frac > 0.f && keep_frac <= 1.f)) return SLR_ERR_ARG;
  int kc, kn;
  if ((st = counts(sh.nb, keep_frac, 0.f, &kc, &kn)) != SLR_OK) return st;
  const bool dense = kc == sh.nb;
  if (!dense && sh.nb > kMaxClassifyBlocks) return SLR_ERR_UNSUPPORTED;
  if ((st = ws_check(ws, ws_bytes, slr_workspace_bytes(SLR_OP_SVOO_ATTN, seq, &keep_frac))) != SLR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve c(ws);
  SvooAttnWs w;
  plan_svoo_attn(c, sh, kc, w);
  SLR_TRY(cudaMemsetAsync(w.status, 0, sizeof(int), s));
  SLR_LAUNCH(kKSvooGather, s, launch_svoo_gather(q, k, v, q_perm, k_perm, w.qp, w.kp, w.vp, sh.BH, sh.d, sh.n_pad,
                                                 w.status, s));
  AttnArgs a = attn_base(sh, w.qp, w.kp, w.vp, w.op, w.status);
  if (dense) {
    if (mask_out_opt) SLR_TRY(cudaMemsetAsync(mask_out_opt, 1, (size_t)sh.BH * sh.nb * sh.nb, s));
  } else {
    SLR_LAUNCH(kKPool, s, launch_pool_means(w.qp, w.kp, w.cls.qsplit, w.cls.ksplit, nullptr, SLR_PHI_ELU1, sh.BH,
                                            sh.d, sh.s, s));
    SLR_LAUNCH(kKLogits, s, launch_logits(w.cls.qsplit, w.cls.ksplit, w.cls.keys, sh.BH, sh.nb, sh.d, w.status, s));
    SLR_LAUNCH(kKClassify, s, launch_classify(w.cls.keys, sh.BH, sh.nb, sh.d, kc, 0, mask_out_opt, nullptr, nullptr,
                                              nullptr, 0, nullptr, w.list, w.list_cnt, w.cap, sh.s, w.status, s));
    a.list = w.list; a.list_cnt = w.list_cnt; a.list_cap = w.cap; a.list_per_head = 1;
  }
  SLR_LAUNCH(kKAttention, s, launch_attention(a, s));
  SLR_LAUNCH(kKSvooScatter, s, launch_svoo_scatter_rows(w.op, q_perm, out, sh.BH, sh.d, sh.n_pad, w.status, s));
  return SLR_OK;
}

}  // extern "C"
