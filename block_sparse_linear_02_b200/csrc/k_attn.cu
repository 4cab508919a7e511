// k_attn.cu -- block-sparse flash attention on tcgen05 (sm_100a).
//
// Computes, for every 64-token query block i, exact softmax attention over the
// valid keys of a set of 64-token key blocks (SLA page section 3, the critical
// branch, which runs block-sparse FlashAttention; the LVSA page's step-6 formula
// is the same normalised sum).  Two fused epilogues:
//   LINEAR  (SLA): the linear-attention branch of the same query block is added,
//           O = O_s + phi(Q_i) H_i' / (phi(Q_i) . Z_i) with H_i' = sum of
//           phi(K_j)^T V_j W_proj over its marginal blocks -- one more MMA of
//           phi(Q) against the H_i'^T rows, and the denominator as a dot product
//           of phi(q) with Z_i in the softmax warps;
//   GATED   (RoPeSLR page): a far-field block of 64 pooled tokens with its own
//           softmax, combined as g*local + (1-g)*far.
//
// A tile is a PAIR of consecutive query blocks (128 query rows = the M of a
// tcgen05 MMA); the kernel is persistent (one CTA per SM takes tiles from a global
// queue) and a tile walks the union of its key-block sets; each list entry
// carries the block's valid-key count and one flag per half of the pair.  The
// list is consumed two entries per STEP (128 keys): one 128x128 S tile per step
// keeps the MMA instruction count and the commits per key low.
// Warp roles (320 threads):
//   warp 8     TMA producer: Q once, then K_0, V_0, K_1, V_1, ... (each item the
//              step's two 64-key blocks) into a 5-slot ring.  With LINEAR the
//              first three slots first hold the two query blocks' linear states
//              and phi(Q), and the K/V items start behind them; without it V_j and
//              K_{j+1} complete one barrier per step;
//   warp 9     MMA issuer: S_j = Q [K_a ; K_b]^T (N = 128) into one of two TMEM
//              S buffers; once both softmax warpgroups have written P_j back
//              over S_j (bf16, in TMEM), O_0 += P_j[:, a] V_a and
//              O_1 += P_j[:, b] V_b with the A operand read from TMEM;
//   warps 0-3  softmax warpgroup 0: the first block of every step;
//   warps 4-7  softmax warpgroup 1: the second block.
// Each warpgroup runs its own online softmax (own running max and sum, own TMEM
// accumulator O_w) over its share of the key blocks; the epilogue merges the two
// shares exactly: O = (2^(m0-M) O_0 + 2^(m1-M) O_1) / (2^(m0-M) l_0 + 2^(m1-M) l_1).
// The softmax works in the exp2 domain with lazy rescaling (an accumulator is
// rescaled only when its running max grows by more than 2^8).  The output leaves
// through shared memory: each softmax warp stages its 32 rows x 32 columns and one TMA
// tensor store writes them (in the tile layout the 32 rows are a 2 x 4 x 4 brick).
#include <cuda_runtime.h>
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace slr {
namespace {

constexpr int kSlots = 5;           // ring of K/V items, each 128 rows x d
constexpr int kThreads = 320;
constexpr uint32_t kColO0 = 0;      // accumulator of warpgroup 0
constexpr uint32_t kColO1 = 128;    // accumulator of warpgroup 1
constexpr uint32_t kColS = 256;     // two 128-column S/P buffers: [256, 384) and [384, 512)

template <int D>
struct AttnLayout {
  static constexpr int kChunks = D / 64;                 // 64-column (128-byte) chunks
  static constexpr int kTile = 128 * 128;                // bytes of one 128-row chunk (Q, or two K/V blocks)
  static constexpr int kHalf = 64 * 128;                 // bytes of one 64-row block inside a chunk
  static constexpr int kKV = kChunks * kTile;            // one ring item: K (or V) of one step
  static constexpr int kHsChunk = D * 128;               // H'^T rows of one query block: D rows per 64-column chunk
  static constexpr int kHsTile = kChunks * kHsChunk;     // one ring item
  static constexpr int kZChunk = 128;                    // the Z row, one 64-column chunk
  static constexpr int kZTile = kChunks * kZChunk;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kChunks * kTile;
  static constexpr int kZOff = kRingOff + kSlots * kKV;  // [2 tile parities][2 query blocks] Z rows
  static constexpr int kXOff = kZOff + 4 * kZTile;       // exchange area: [2 shares][2 tiles][3][128] floats
  static constexpr int kBarOff = kXOff + 12 * 128 * 4;
  // output staging: per softmax warp one 32-row x 32-column bf16 chunk (64-byte rows,
  // 64-byte swizzle), written to HBM by TMA tensor stores
  static constexpr int kOutChunk = 32 * 64;
  static constexpr int kOutOff = (kBarOff + 512 + 1023) / 1024 * 1024;
  static constexpr int kBytes = kOutOff + 8 * kOutChunk + 1024;   // + alignment slack
  static_assert(kHsTile <= kKV, "a linear state tile must fit in one ring slot");
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
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
  int n_tiles;            // heads x pairs
  int* tile_counter;      // global tile queue, zero at launch
};

constexpr int kTq = 4;    // tile-index slots between the producer and the other roles

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

// Paired fp32 arithmetic: one instruction does the work of two, rounded as the scalar forms.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// D[tmem] (+)= A[tmem] * B[smem]^T (A: row m in lane m, two bf16 of K per column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
               :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
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

// List word: key block in bits [0,16), valid keys in bits [16,23), bit 30/31: half 0/1
// attends.  The softmax side needs the valid-key count and the two attend bits.
struct Entry {
  int nvalid;
  uint32_t flags;
};

// Per-tile quantities every role derives from the tile index.
struct TileInfo {
  int bh, pair;
  const uint32_t* list;            // null = every key block (dense)
  int n_local, local_steps, n_steps, n_lin;
  bool second_exists;
};

template <bool GATED, bool LINEAR>
__device__ __forceinline__ TileInfo tile_info(int t, const AttnKParams& p) {
  TileInfo ti;
  ti.bh = t / p.n_pairs;
  ti.pair = t % p.n_pairs;
  ti.list = nullptr;
  ti.n_local = p.n_kb;
  if (p.list) {
    const size_t off = (p.list_per_head ? (size_t)ti.bh * p.n_pairs : 0) + ti.pair;
    ti.list = p.list + off * p.list_cap;
    ti.n_local = p.list_cnt[off];
  }
  ti.local_steps = (ti.n_local + 1) >> 1;
  ti.n_steps = ti.local_steps + (GATED ? 1 : 0);   // the far block is a step of its own
  ti.second_exists = 2 * ti.pair + 1 < p.n_qb;
  ti.n_lin = LINEAR ? (ti.second_exists ? 2 : 1) : 0;
  return ti;
}

// Persistent: one CTA per SM takes tiles (head, pair of query blocks) from a global
// queue.  The producer fetches the next tile index as soon as it has issued the current
// tile's loads and hands it to the other roles through a small ring of tile slots, so
// the next tile's Q, linear states and first K/V blocks load while the current tile
// finishes.  Ring positions, step counters and the per-tile barriers run on across tiles.
template <int D, bool TILE, bool GATED, bool LINEAR>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmX1,
            const __grid_constant__ CUtensorMap tmX2, const __grid_constant__ CUtensorMap tmX3,
            const __grid_constant__ CUtensorMap tmO, const AttnKParams p) {
  // tmX1/tmX2: far-field K/V maps (GATED), or the linear state maps (LINEAR): tmX1 the
  // H'^T rows (box D rows), tmX2 the Z row with 15 rows of zero fill (box 16 rows);
  // tmX3: phi(Q) (LINEAR, same boxes as Q).  tmO: the output, boxes of 32 rows x 32
  // columns with 64-byte swizzle; in the tile layout the 32 rows are a 2 x 4 x 4
  // (frame, height, width) brick of one 4 x 4 x 4 tile.
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sRing = smem + L::kRingOff;
  uint8_t* sZ = smem + L::kZOff;
  float* xch = reinterpret_cast<float*>(smem + L::kXOff);   // [2 tiles][3][128]: m, l, far-l per warpgroup share
  uint8_t* sOut = smem + L::kOutOff;                         // [8 softmax warps] output staging chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;                   // Q of the current tile landed
  uint64_t* q_free = q_full + 1;                 // every MMA reading Q of a tile has completed
  uint64_t* slot_full = q_free + 1;              // [kSlots] ring slot filled (TMA, or freed for phi(Q))
  uint64_t* s_full = slot_full + kSlots;         // [4] per step mod 4: S_j written (the step's K item is free)
  uint64_t* p_full = s_full + 4;                 // [2] per S buffer, 256 arrivals
  uint64_t* pv_done = p_full + 2;                // [4] per step mod 4 (phases cannot alias)
  uint64_t* den_done = pv_done + 4;              // the tile's phi(Q) slot has been read (256 arrivals per tile)
  uint64_t* lin_done = den_done + 1;
  uint64_t* lin_read = lin_done + 1;             // the tile's linear result has been read (256 arrivals per tile)
  uint64_t* o_free = lin_read + 1;               // the epilogue has read O_0/O_1 (256 arrivals per tile)
  uint64_t* xch_bar = o_free + 1;                // both shares of every row published (256 arrivals per tile)
  uint64_t* tq_full = xch_bar + 1;               // [kTq] tile slot written
  uint64_t* tq_empty = tq_full + kTq;            // [kTq] tile slot read (MMA thread + one lane per softmax warp)
  uint64_t* drain = tq_empty + kTq;
  uint64_t* kv_step = drain + 1;                 // [4] per step mod 4: V_j and K_{j+1} landed (non-LINEAR)
  uint64_t* z_full = kv_step + 4;                // [2] per tile parity: the tile's Z rows landed (LINEAR)
  int* tq = reinterpret_cast<int*>(z_full + 2);  // [kTq] tile indices
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq + kTq);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 512;
  const SeqShape seq{p.n_pad, p.seg_len, p.seg_stride, p.n_kb};
  // LINEAR: a tile's first three ring positions hold the H'^T rows of its two query
  // blocks and phi(Q); its K/V items follow
  constexpr int kPre = LINEAR ? 3 : 0;
  // Without the linear pre-slots the ring positions of a tile's items are regular, and
  // V_j and K_{j+1} (consecutive positions) complete one step barrier together, so the MMA
  // thread polls once per step for both.  Their slots are freed by step j-2 (K_{j-2}'s QK,
  // V_{j-2}'s P.V), so waiting for both before issuing either delays only V_j, which is not
  // needed before P.V_j.
  constexpr bool KVSTEP = !LINEAR;
  // LINEAR: the tile's lin = phi(Q) H'_b (D columns) is written into the S buffer that step 1
  // of the tile will use, so it waits neither for the previous tile's epilogue nor for O

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int s = 0; s < kSlots; ++s) mbar_init(&slot_full[s], 1);
    for (int b = 0; b < 4; ++b) mbar_init(&s_full[b], 1);
    for (int b = 0; b < 2; ++b) mbar_init(&p_full[b], 256);
    for (int b = 0; b < 4; ++b) mbar_init(&pv_done[b], 1);
    mbar_init(den_done, 256);
    mbar_init(lin_done, 1);
    mbar_init(lin_read, 256);
    mbar_init(o_free, 256);
    mbar_init(xch_bar, 256);
    for (int e = 0; e < kTq; ++e) { mbar_init(&tq_full[e], 1); mbar_init(&tq_empty[e], 9); }
    mbar_init(drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&kv_step[q], 1);
    for (int q = 0; q < 2; ++q) mbar_init(&z_full[q], 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      // how the current occupant of each ring slot is released: kind 0 = the P.V of
      // global step idx (a V item), kind 3 = the QK of global step idx (a K item: only QK
      // reads it, so its slot turns over a step earlier, which lets the next tile's first
      // K load while the current tile still runs), kind 1 = the linear-branch MMAs of
      // local tile idx, kind 2 = those MMAs and the softmax warps' denominator reads of
      // local tile idx, -1 = free
      int rel_kind[kSlots], rel_idx[kSlots];
      #pragma unroll
      for (int s = 0; s < kSlots; ++s) { rel_kind[s] = -1; rel_idx[s] = 0; }
      auto slot_released = [&](int slot) -> bool {
        if (rel_kind[slot] == 0) {
          const int q = rel_idx[slot];
          return mbar_wait(&pv_done[q & 3], (q >> 2) & 1, abort_flag, p.status);
        }
        if (rel_kind[slot] == 3) {
          const int q = rel_idx[slot];
          return mbar_wait(&s_full[q & 3], (q >> 2) & 1, abort_flag, p.status);
        }
        if (rel_kind[slot] >= 1) {
          if (!mbar_wait(lin_done, rel_idx[slot] & 1, abort_flag, p.status)) return false;
          if (rel_kind[slot] == 2) return mbar_wait(den_done, rel_idx[slot] & 1, abort_flag, p.status);
        }
        return true;
      };
      int i = 0, J = 0, g = 0, q_loaded = -1, kv_armed = -1;   // kv_armed: last step barrier armed
      bool ok = true;
      int t_next = atomicAdd(p.tile_counter, 1);       // the queue is read one tile ahead
      while (ok) {
        int t = t_next;
        if (t > p.n_tiles) t = p.n_tiles;              // sentinel: no more tiles
        if (t < p.n_tiles) t_next = atomicAdd(p.tile_counter, 1);
        const int e = i % kTq;
        if (i >= kTq && !(ok = mbar_wait(&tq_empty[e], ((i / kTq) - 1) & 1, abort_flag, p.status))) break;
        tq[e] = t;
        mbar_arrive(&tq_full[e]);
        if (t >= p.n_tiles) break;
        const TileInfo ti = tile_info<GATED, LINEAR>(t, p);
        auto step_blocks = [&](int j) -> int {
          if (GATED && j == ti.local_steps) return 1;
          return (2 * j + 1 < ti.n_local) ? 2 : 1;
        };
        // Q of this tile once every MMA of the previous tile that reads it is done
        if (i > 0 && !(ok = mbar_wait(q_free, (i - 1) & 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(q_full, L::kChunks * L::kTile);
        q_loaded = i;
        if (TILE) {
          for (int half = 0; half < 2; ++half) {
            int tf, th, tw;
            tile_coords(2 * ti.pair + half, p.TF, p.TW, tf, th, tw);
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_5d(sQ + c * L::kTile + half * L::kHalf, &tmQ, q_full, c * 64, tw * 4, th * 4, tf * 4, ti.bh);
          }
        } else {
          for (int c = 0; c < L::kChunks; ++c) tma_load_3d(sQ + c * L::kTile, &tmQ, q_full, c * 64, ti.pair * 128, ti.bh);
        }
        if (LINEAR) {
          // row D of the state (Z) of each query block, into this tile parity's buffer and on the
          // parity's own barrier: the softmax warps read it at the tile start, which can come
          // after the next tile's Q has landed (a one-step tile releases Q after its only QK),
          // so neither the buffer nor q_full's phase may be shared with the next tile
          mbar_arrive_expect_tx(&z_full[i & 1], ti.n_lin * L::kZTile);
          for (int b = 0; b < ti.n_lin; ++b)
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_3d(sZ + ((i & 1) * 2 + b) * L::kZTile + c * L::kZChunk, &tmX2, &z_full[i & 1], c * 64, D,
                          ti.bh * p.n_qb + 2 * ti.pair + b);
        }
        if (LINEAR) {
          // pre-slots by TMA: the states of the two query blocks, then phi(Q); a missing
          // second query block's slot completes its phase with a plain arrive
          for (int pr = 0; pr < 3 && ok; ++pr, ++g) {
            const int slot = g % kSlots;
            if (!(ok = slot_released(slot))) break;
            if (pr == 2) {
              mbar_arrive_expect_tx(&slot_full[slot], L::kChunks * L::kTile);
              for (int c = 0; c < L::kChunks; ++c)
                tma_load_3d(sRing + slot * L::kKV + c * L::kTile, &tmX3, &slot_full[slot], c * 64, ti.pair * 128, ti.bh);
            } else if (pr < ti.n_lin) {
              mbar_arrive_expect_tx(&slot_full[slot], L::kHsTile);
              for (int c = 0; c < L::kChunks; ++c)
                tma_load_3d(sRing + slot * L::kKV + c * L::kHsChunk, &tmX1, &slot_full[slot], c * 64, 0,
                            ti.bh * p.n_qb + 2 * ti.pair + pr);
            } else {
              mbar_arrive(&slot_full[slot]);
            }
            rel_kind[slot] = pr == 2 ? 2 : 1;
            rel_idx[slot] = i;
          }
        }
        // one K or V item of step j into a ring slot, its TMA completing on barrier `bar`
        auto load_item = [&](int slot, int j, bool is_v, uint64_t* bar) {
          const int nb = step_blocks(j);
          const bool far = GATED && j == ti.local_steps;
          for (int b = 0; b < nb; ++b) {
            uint8_t* dst = sRing + slot * L::kKV + b * L::kHalf;
            if (far) {
              for (int c = 0; c < L::kChunks; ++c)
                tma_load_3d(dst + c * L::kTile, is_v ? &tmX2 : &tmX1, bar, c * 64, 0, ti.bh);
            } else {
              // key block kb: rows [64 kb, 64 kb + 64) (in the tile layout K and V are in
              // tile-major order, so a 4x4x4 tile is one such block)
              const int kb = ti.list ? (int)(ti.list[2 * j + b] & 0xFFFFu) : 2 * j + b;
              const CUtensorMap* tm = is_v ? &tmV : &tmK;
              for (int c = 0; c < L::kChunks; ++c)
                tma_load_3d(dst + c * L::kTile, tm, bar, c * 64, kb * 64, ti.bh);
            }
          }
        };
        auto item_bytes = [&](int j) -> uint32_t { return (uint32_t)(step_blocks(j) * L::kChunks * L::kHalf); };
        if (KVSTEP) {
          // K_0 on its slot barrier; then per step j, V_j and K_{j+1} on kv_step[j]; their slot
          // barriers get a plain arrive, so every use of a slot still advances its phase once
          if (ti.n_steps > 0 && ok) {
            const int slot = g % kSlots;
            if ((ok = slot_released(slot))) {
              mbar_arrive_expect_tx(&slot_full[slot], item_bytes(0));
              load_item(slot, 0, false, &slot_full[slot]);
              rel_kind[slot] = 3;
              rel_idx[slot] = J;
              ++g;
            }
          }
          for (int j = 0; j < ti.n_steps && ok; ++j) {
            const bool has_k = j + 1 < ti.n_steps;
            const int sv = g % kSlots, sk = (g + 1) % kSlots;
            if (!(ok = slot_released(sv))) break;
            if (has_k && !(ok = slot_released(sk))) break;
            uint64_t* bar = &kv_step[(J + j) & 3];
            mbar_arrive_expect_tx(bar, item_bytes(j) + (has_k ? item_bytes(j + 1) : 0u));
            load_item(sv, j, true, bar);
            mbar_arrive(&slot_full[sv]);
            rel_kind[sv] = 0;
            rel_idx[sv] = J + j;
            ++g;
            if (has_k) {
              load_item(sk, j + 1, false, bar);
              mbar_arrive(&slot_full[sk]);
              rel_kind[sk] = 3;
              rel_idx[sk] = J + j + 1;
              ++g;
            }
            kv_armed = J + j;
          }
        } else {
          // K/V items: K (even it) or V (odd it) of step it/2
          for (int it = 0; it < 2 * ti.n_steps && ok; ++it, ++g) {
            const int slot = g % kSlots;
            if (!(ok = slot_released(slot))) break;
            const int j = it >> 1;
            const bool is_v = it & 1;
            mbar_arrive_expect_tx(&slot_full[slot], item_bytes(j));
            load_item(slot, j, is_v, &slot_full[slot]);
            rel_kind[slot] = is_v ? 0 : 3;
            rel_idx[slot] = J + j;
          }
        }
        J += ti.n_steps;
        ++i;
      }
      if (*abort_flag) {
        // let the loads already in flight land before the CTA's shared memory is released
        long long t0 = clock64();
        if (q_loaded >= 0) while (!mbar_try_wait(q_full, q_loaded & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        if (LINEAR && q_loaded >= 0) {
          t0 = clock64();
          while (!mbar_try_wait(&z_full[q_loaded & 1], (q_loaded >> 1) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
        for (int gg = (g - kSlots > 0 ? g - kSlots : 0); gg < g; ++gg) {
          t0 = clock64();
          while (!mbar_try_wait(&slot_full[gg % kSlots], (gg / kSlots) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
        // the step barriers whose loads may still be in flight (the ring holds at most 3 steps)
        for (int q = (kv_armed - 3 > 0 ? kv_armed - 3 : 0); q <= kv_armed; ++q) {
          t0 = clock64();
          while (!mbar_try_wait(&kv_step[q & 3], (q >> 2) & 1) && clock64() - t0 < kWaitBudgetCycles) {}
        }
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), ring_addr = smem_u32(sRing);
      // Shared-memory descriptors: the start-address field is (address >> 4) in the low 14
      // bits and every operand lies below 256 KB, so an operand's descriptor is a base
      // descriptor plus its byte offset >> 4.
      const uint64_t dQ = desc_kmajor(q_addr);
      const uint64_t dK = desc_kmajor(ring_addr);
      const uint64_t dV = desc_mnmajor(ring_addr, L::kTile);
      auto issue_qk = [&](int slot, int sbuf) {
        const uint64_t db = dK + (uint32_t)((slot * L::kKV) >> 4);
        #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(((kk >> 2) * L::kTile + (kk & 3) * 32) >> 4);
          mma_bf16_ss(tmem + kColS + sbuf * 128, dQ + off, db + off, idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_dst (+)= P[:, 64*blk .. +64] V_blk; P lives in TMEM over the step's S buffer
      auto issue_pv = [&](int slot, int sbuf, int blk, uint32_t col, bool acc) {
        const uint64_t db = dV + (uint32_t)((slot * L::kKV + blk * L::kHalf) >> 4);
        const uint32_t a = tmem + kColS + sbuf * 128 + blk * 64;
        #pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + col, a + kk * 8, db + (uint32_t)(kk * 2048 >> 4), idO, (acc || kk > 0) ? 1u : 0u);
      };
      // lin = phi(Q) H'_b per query block b (lanes of the other block masked off) into the
      // TMEM columns col (the S buffer of the tile's step 1); the denominators phi(q) . Z_b
      // are dot products the softmax warps form from phi(Q) in shared memory
      auto issue_lin = [&](int g0, int n_lin, uint32_t col) {
        constexpr uint32_t idH = idesc_bf16(128, D, false, false);
        const uint32_t phq_addr = ring_addr + ((g0 + 2) % kSlots) * L::kKV;
        const uint32_t lo_only[4] = {0u, 0u, 0xFFFFFFFFu, 0xFFFFFFFFu};   // write lanes 0-63
        const uint32_t hi_only[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0u, 0u};   // write lanes 64-127
        for (int b = 0; b < n_lin; ++b) {
          const uint32_t hs_addr = ring_addr + ((g0 + b) % kSlots) * L::kKV;
          #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int c = kk >> 2, sub = kk & 3;
            const uint64_t a = desc_kmajor(phq_addr + c * L::kTile + sub * 32);
            const uint64_t bh_ = desc_kmajor(hs_addr + c * L::kHsChunk + sub * 32);
            mma_bf16_ss_masked(tmem + col, a, bh_, idH, kk > 0 ? 1u : 0u, b ? hi_only : lo_only);
          }
        }
        mma_commit(lin_done);
      };
      // LINEAR: the local tile whose linear result the softmax warps may still be reading
      // from an S buffer; any MMA that writes an S buffer first waits for that read
      int lin_tile = -1;
      auto settle_lin = [&]() -> bool {
        if (!LINEAR || lin_tile < 0) return true;
        const int tl = lin_tile;
        lin_tile = -1;
        return mbar_wait(lin_read, tl & 1, abort_flag, p.status);
      };
      int i = 0, J = 0, g = 0;
      bool ok = true;
      while (ok) {
        const int e = i % kTq;
        if (!(ok = mbar_wait(&tq_full[e], (i / kTq) & 1, abort_flag, p.status))) break;
        const int t = tq[e];
        mbar_arrive(&tq_empty[e]);
        if (t >= p.n_tiles) break;
        const TileInfo ti = tile_info<GATED, LINEAR>(t, p);
        auto step_blocks = [&](int j) -> int {
          if (GATED && j == ti.local_steps) return 1;
          return (2 * j + 1 < ti.n_local) ? 2 : 1;
        };
        const int gkv = g + kPre;                  // ring position of this tile's K_0
        if (LINEAR) {
          // lin first: it needs only the pre-slots (loaded ahead of K_0), and the softmax
          // warps read it while QK_0 runs.  Its S buffer was last read by the P.V of the
          // previous tile's last step, issued earlier from this thread (MMAs run in order).
          ok = mbar_wait(&slot_full[(g + 2) % kSlots], ((g + 2) / kSlots) & 1, abort_flag, p.status) &&
               mbar_wait(&slot_full[g % kSlots], (g / kSlots) & 1, abort_flag, p.status) &&
               mbar_wait(&slot_full[(g + 1) % kSlots], ((g + 1) / kSlots) & 1, abort_flag, p.status) &&
               settle_lin();
          if (!ok) break;
          tc_fence_after();
          issue_lin(g, ti.n_lin, kColS + ((J + 1) & 1) * 128);
          lin_tile = i;
        }
        if (!(ok = mbar_wait(q_full, i & 1, abort_flag, p.status))) break;
        // GATED: the previous tile's far-field output sits in the S buffer this tile's
        // first QK writes, so wait until its epilogue has read it
        if (GATED && i > 0 && !(ok = mbar_wait(o_free, (i - 1) & 1, abort_flag, p.status))) break;
        if (ti.n_steps > 0) {
          if (!(ok = mbar_wait(&slot_full[gkv % kSlots], (gkv / kSlots) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_qk(gkv % kSlots, J & 1);           // S buffer J & 1: never the tile's lin buffer
          mma_commit(&s_full[J & 3]);
        }
        if (ti.n_steps <= 1) mma_commit(q_free);   // the last MMA reading Q has been issued
        bool o1_started = false;
        for (int j = 0; j < ti.n_steps && ok; ++j) {
          const int Jj = J + j, b = Jj & 1;
          if (KVSTEP) {                            // V_j and K_{j+1} have landed (one barrier for both)
            if (!(ok = mbar_wait(&kv_step[Jj & 3], (Jj >> 2) & 1, abort_flag, p.status))) break;
            tc_fence_after();
          }
          if (j + 1 < ti.n_steps) {
            const int gk = gkv + 2 * (j + 1);
            ok = KVSTEP || mbar_wait(&slot_full[gk % kSlots], (gk / kSlots) & 1, abort_flag, p.status);
            if (!(ok = ok && settle_lin())) break;
            tc_fence_after();
            issue_qk(gk % kSlots, (Jj + 1) & 1);
            mma_commit(&s_full[(Jj + 1) & 3]);
            if (j + 2 == ti.n_steps) mma_commit(q_free);
          }
          const int gv = gkv + 2 * j + 1;
          if ((!KVSTEP && !mbar_wait(&slot_full[gv % kSlots], (gv / kSlots) & 1, abort_flag, p.status)) ||
              !mbar_wait(&p_full[b], (Jj >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const bool far = GATED && j == ti.local_steps;
          if (far) {
            // the far-field output goes into the other S buffer (its step is done)
            issue_pv(gv % kSlots, b, 0, kColS + (b ^ 1) * 128, false);
          } else {
            issue_pv(gv % kSlots, b, 0, kColO0, j > 0);
            if (step_blocks(j) == 2) {
              issue_pv(gv % kSlots, b, 1, kColO1, o1_started);
              o1_started = true;
            }
          }
          mma_commit(&pv_done[Jj & 3]);
        }
        g += kPre + 2 * ti.n_steps;
        J += ti.n_steps;
        ++i;
      }
      if (!ok) {
        mma_commit(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int wg = warp >> 2;                  // 0: first block of a step, 1: second block
    const int r = threadIdx.x & 127;           // query row of the pair = TMEM lane
    const int half = r >> 6;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t my_o = wg ? kColO1 : kColO0;
    const float sl = p.scale_log2;
    int i = 0, J = 0, g = 0;
    bool ok = true;
    while (ok) {
      const int e = i % kTq;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tq_full[e], (i / kTq) & 1, abort_flag, p.status));
      if (!ok) break;
      const int t = tq[e];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tq_empty[e]);
      if (t >= p.n_tiles) break;
      const TileInfo ti = tile_info<GATED, LINEAR>(t, p);
      const int local_steps = ti.local_steps, n_steps = ti.n_steps, n_local = ti.n_local;
      auto step_blocks = [&](int j) -> int {
        if (GATED && j == local_steps) return 1;
        return (2 * j + 1 < n_local) ? 2 : 1;
      };
      float m_run = -INFINITY, l_run = 0.f, l_far = 0.f;
      bool started = false;

      // ---- token of this row
      int tok;
      bool row_exists;
      if (TILE) {
        const int tile = 2 * ti.pair + half;
        row_exists = tile < p.n_qb;
        int tf, th, tw;
        tile_coords(tile, p.TF, p.TW, tf, th, tw);
        const int rr = r & 63;
        tok = ((tf * 4 + (rr >> 4)) * p.Hh + th * 4 + ((rr >> 2) & 3)) * p.Ww + tw * 4 + (rr & 3);
      } else {
        tok = ti.pair * 128 + r;
        row_exists = tok < p.n_pad;
      }
      const bool valid = row_exists && (TILE || token_valid(seq, tok));

      // ---- linear branch (LINEAR): phi(Q) arrives by TMA in the tile's third pre-slot, and
      // the MMA warp's lin = phi(Q) H'_b lands in the S buffer of the tile's step 1; my half
      // of the row is read before the first step (the QK of step 1 waits for that read) and
      // kept in registers as bf16 pairs (the output is rounded to bf16 in the end as well).
      // The denominator phi(q) . Z_b is a dot product over the same bf16 phi values, my half
      // of the channels here, summed with the other half in the epilogue.
      uint32_t lin[D / 4];
      #pragma unroll
      for (int k = 0; k < D / 4; ++k) lin[k] = 0u;
      float den_part = 0.f;
      if (LINEAR) {
        const int gphi = g + 2;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&z_full[i & 1], (i >> 1) & 1, abort_flag, p.status) &&
                                         mbar_wait(&slot_full[gphi % kSlots], (gphi / kSlots) & 1, abort_flag, p.status));
        if (ok) {
          const uint8_t* sPhi = sRing + (gphi % kSlots) * L::kKV;
          const uint8_t* zrow = sZ + ((i & 1) * 2 + half) * L::kZTile;   // Z of my query block, this tile parity
          constexpr int kGroups = D / 16;                  // 16-byte groups of my row handled by my warpgroup
          #pragma unroll
          for (int gr = 0; gr < kGroups; ++gr) {
            const int gg = wg * kGroups + gr;              // 0 .. D/8-1
            const uint4 u = *reinterpret_cast<const uint4*>(sPhi + (gg >> 3) * L::kTile + sw128_offset(r, gg & 7));
            const uint4 zu = *reinterpret_cast<const uint4*>(zrow + (gg >> 3) * L::kZChunk + (gg & 7) * 16);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            const uint32_t zw[4] = {zu.x, zu.y, zu.z, zu.w};
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
              den_part = fmaf(bf16_lo(w[k]), bf16_lo(zw[k]), den_part);
              den_part = fmaf(bf16_hi(w[k]), bf16_hi(zw[k]), den_part);
            }
          }
        }
        mbar_arrive(den_done);
        if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(lin_done, i & 1, abort_flag, p.status));
        tc_fence_after();
        if (ok) {
          const uint32_t lin_addr = lane_addr + kColS + ((J + 1) & 1) * 128 + wg * (D / 2);
          #pragma unroll
          for (int k = 0; k < D / 64; ++k) {
            uint32_t tv[32];
            tmem_ld32(lin_addr + k * 32, tv);
            tmem_wait_ld();
            #pragma unroll
            for (int m = 0; m < 16; ++m) lin[k * 16 + m] = pack_bf16(__uint_as_float(tv[2 * m]), __uint_as_float(tv[2 * m + 1]));
          }
          tc_fence_before();
          mbar_arrive(lin_read);
        }
      }

      // my list word of step j, loaded one step ahead and decoded only where it is used, so
      // that the load's latency is not waited for at the top of the step
      auto word_of = [&](int j) -> uint32_t {
        const bool far_j = GATED && j == local_steps;
        if (ti.list && j < n_steps && !far_j && (wg == 0 || step_blocks(j) == 2)) return ti.list[2 * j + wg];
        return 0u;
      };
      uint32_t w_next = word_of(0);
      for (int j = 0; j < n_steps && ok; ++j) {
        const int Jj = J + j, b = Jj & 1;
        const bool far = GATED && j == local_steps;
        const bool mine = wg == 0 || (!far && step_blocks(j) == 2);   // does this warpgroup own a block here
        const uint32_t w_cur = w_next;
        w_next = word_of(j + 1);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[Jj & 3], (Jj >> 2) & 1, abort_flag, p.status))) { ok = false; break; }
        tc_fence_after();
        if (!mine) {
          tc_fence_before();
          mbar_arrive(&p_full[b]);
          continue;
        }
        const uint32_t s_addr = lane_addr + kColS + b * 128 + wg * 64;
        uint32_t sr[64];
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        Entry en{64, 3u};
        if (!far) {
          if (ti.list) {
            en.nvalid = (int)((w_cur >> 16) & 0x7Fu);
            en.flags = w_cur >> 30;
          } else if (!TILE) {
            en.nvalid = block_valid_count(seq, 2 * j + wg);
          }
        }
        const bool attend = (en.flags >> half) & 1u;
        const int nvalid = attend ? en.nvalid : 0;
        tmem_wait_ld();
        // A full block against a running max already set: exponentials against that max
        // with the row max taken in the same pass; only a row whose max then rises past
        // the lazy-rescale threshold repeats the pass (the same P as with the max first).
        // Not in the LINEAR variant, which holds the linear result in registers and ran
        // slower with the fused pass.
        const bool spec = !LINEAR && !far && nvalid == 64 && m_run != -INFINITY;
        float mx = -INFINITY;
        uint32_t packed[32];
        float rowsum = 0.f;
        if (spec) {
          const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_run, -m_run);
          float2 acc = make_float2(0.f, 0.f);
          float mx0 = -INFINITY, mx1 = -INFINITY;
          #pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float s0 = __uint_as_float(sr[c]), s1 = __uint_as_float(sr[c + 1]);
            const float s2 = __uint_as_float(sr[c + 2]), s3 = __uint_as_float(sr[c + 3]);
            const float2 x01 = fma2(make_float2(s0, s1), sl2, nm2), x23 = fma2(make_float2(s2, s3), sl2, nm2);
            const float p0 = ex2(x01.x), p1 = ex2(x01.y), p2 = ex2(x23.x), p3 = ex2(x23.y);
            acc = add2(acc, add2(make_float2(p0, p1), make_float2(p2, p3)));
            packed[c >> 1] = pack_bf16(p0, p1);
            packed[(c >> 1) + 1] = pack_bf16(p2, p3);
            mx0 = max3(mx0, s0, s1);
            mx1 = max3(mx1, s2, s3);
          }
          rowsum = acc.x + acc.y;
          mx = fmaxf(mx0, mx1);
        } else if (nvalid == 64) {
          float t3[22];
          #pragma unroll
          for (int k = 0; k < 21; ++k)
            t3[k] = max3(__uint_as_float(sr[3 * k]), __uint_as_float(sr[3 * k + 1]), __uint_as_float(sr[3 * k + 2]));
          t3[21] = __uint_as_float(sr[63]);
          float u[8];
          #pragma unroll
          for (int k = 0; k < 7; ++k) u[k] = max3(t3[3 * k], t3[3 * k + 1], t3[3 * k + 2]);
          u[7] = t3[21];
          mx = fmaxf(max3(u[0], u[1], u[2]), max3(max3(u[3], u[4], u[5]), u[6], u[7]));
        } else if (nvalid > 0) {
          #pragma unroll
          for (int c = 0; c < 64; ++c) {
            if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
            mx = fmaxf(mx, __uint_as_float(sr[c]));
          }
        }
        // far step: a fresh softmax of its own; local steps: lazy rescale of the running state
        float mu;
        bool need = false;
        float factor = 1.f;
        if (far) {
          mu = mx * sl;
        } else {
          const float m_new = fmaxf(m_run, mx * sl);
          need = m_new > m_run + 8.f;
          if (need) {
            factor = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
            l_run *= factor;
            m_run = m_new;
          }
          mu = m_run;
        }
        if (mu == -INFINITY) mu = 0.f;
        if (!spec || need) {
          rowsum = 0.f;
          if (nvalid == 0) {
            #pragma unroll
            for (int c = 0; c < 32; ++c) packed[c] = 0u;
          } else {
            const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-mu, -mu);
            float2 acc = make_float2(0.f, 0.f);
            #pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 x = fma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2, nm2);
              const float p0 = ex2(x.x), p1 = ex2(x.y);
              acc = add2(acc, make_float2(p0, p1));
              packed[c >> 1] = pack_bf16(p0, p1);
            }
            rowsum = acc.x + acc.y;
          }
        }
        if (far) l_far = rowsum; else l_run += rowsum;
        // rescale my accumulator (once it holds data) after the previous P.V has completed
        if (!far && started && __any_sync(0xFFFFFFFFu, need)) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&pv_done[(Jj - 1) & 3], ((Jj - 1) >> 2) & 1, abort_flag, p.status))) { ok = false; break; }
          tc_fence_after();
          #pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(lane_addr + my_o + cc * 32, o);
            tmem_wait_ld();
            #pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * factor);
            tmem_st32(lane_addr + my_o + cc * 32, o);
          }
        }
        tmem_st32(s_addr, packed);          // P (bf16 pairs) over the first 32 columns of my S block
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
        if (!far) started = true;
      }
      if (ok && n_steps > 0) {
        const int Jl = J + n_steps - 1;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&pv_done[Jl & 3], (Jl >> 2) & 1, abort_flag, p.status));
      }
      ok = __all_sync(0xFFFFFFFFu, ok);
      tc_fence_after();

      // ---- merge the two shares (published through shared memory, double-buffered by tile)
      float* xb = xch + (i & 1) * (3 * 128);
      if (wg == 0) { xb[r] = m_run; xb[128 + r] = l_run; }
      float* xo = xch + 2 * (3 * 128) + (i & 1) * (3 * 128);   // the second warpgroup's share
      if (wg == 1) { xo[r] = m_run; xo[128 + r] = l_run; }
      if (GATED && wg == 0) xb[256 + r] = l_far;
      if (LINEAR) (wg ? xo : xb)[256 + r] = den_part;
      mbar_arrive(xch_bar);
      if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(xch_bar, i & 1, abort_flag, p.status));
      const float m0 = xb[r], l0 = xb[128 + r], m1 = xo[r], l1 = xo[128 + r];
      const float M = fmaxf(m0, m1);
      const float a0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
      const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
      const float Lsum = a0 * l0 + a1 * l1;
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      const float c0 = a0 * inv, c1 = a1 * inv;
      float inv_den = 0.f;
      if (LINEAR) {
        const float den = xb[256 + r] + xo[256 + r];
        inv_den = den > 0.f ? 1.f / den : 0.f;
      }
      float inv_far = 0.f;
      uint32_t col_far = 0;
      if (GATED) {
        const float lf = xb[256 + r];
        inv_far = lf > 0.f ? 1.f / lf : 0.f;
        col_far = kColS + (((J + local_steps) & 1) ^ 1) * 128;
      }
      const bool have_o0 = ok && n_local > 0;        // uniform over the softmax warps
      const bool have_o1 = ok && n_local > 1;
      #pragma unroll
      for (int k = 0; k < D / 64; ++k) {
        const int cc = wg * (D / 64) + k;          // my 32-column chunks
        float v[32];
        #pragma unroll
        for (int m = 0; m < 32; ++m) v[m] = 0.f;
        if (have_o1) {                             // both accumulators, one wait
          uint32_t o0[32], o1[32];
          tmem_ld32(lane_addr + kColO0 + cc * 32, o0);
          tmem_ld32(lane_addr + kColO1 + cc * 32, o1);
          tmem_wait_ld();
          #pragma unroll
          for (int m = 0; m < 32; ++m) v[m] = fmaf(c1, __uint_as_float(o1[m]), c0 * __uint_as_float(o0[m]));
        } else if (have_o0) {
          uint32_t o0[32];
          tmem_ld32(lane_addr + kColO0 + cc * 32, o0);
          tmem_wait_ld();
          #pragma unroll
          for (int m = 0; m < 32; ++m) v[m] = c0 * __uint_as_float(o0[m]);
        }
        if (GATED && ok) {
          uint32_t of[32];
          tmem_ld32(lane_addr + col_far + cc * 32, of);
          tmem_wait_ld();
          #pragma unroll
          for (int m = 0; m < 32; ++m) v[m] = p.gate * v[m] + (1.f - p.gate) * (__uint_as_float(of[m]) * inv_far);
        }
        if (LINEAR) {
          #pragma unroll
          for (int m = 0; m < 16; ++m) {
            v[2 * m] = fmaf(bf16_lo(lin[k * 16 + m]), inv_den, v[2 * m]);
            v[2 * m + 1] = fmaf(bf16_hi(lin[k * 16 + m]), inv_den, v[2 * m + 1]);
          }
        }
        // my row's 32 columns into the warp's staging chunk (64-byte swizzle: 16-byte piece
        // m of row r sits at piece m ^ ((r >> 1) & 3)), then one TMA store of the warp's 32
        // rows; rows past the sequence end are clipped by the tensor map
        uint8_t* stg = sOut + warp * L::kOutChunk;
        if (lane == 0) bulk_wait_read_all();       // the last store from this chunk has read it
        __syncwarp();
        #pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint4 w4 = make_uint4(0, 0, 0, 0);
          if (valid)
            w4 = make_uint4(pack_bf16(v[8 * m], v[8 * m + 1]), pack_bf16(v[8 * m + 2], v[8 * m + 3]),
                            pack_bf16(v[8 * m + 4], v[8 * m + 5]), pack_bf16(v[8 * m + 6], v[8 * m + 7]));
          *reinterpret_cast<uint4*>(stg + lane * 64 + ((m ^ ((lane >> 1) & 3)) << 4)) = w4;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (TILE) {
            // warps 0-1 hold the first tile of the pair, 2-3 the second; each covers two of
            // the tile's four frames (row = 16 f + 4 h + w inside the tile)
            const int tile = 2 * ti.pair + ((warp & 3) >> 1);
            if (tile < p.n_qb) {
              int tf, th, tw;
              tile_coords(tile, p.TF, p.TW, tf, th, tw);
              tma_store_5d(&tmO, stg, cc * 32, tw * 4, th * 4, tf * 4 + 2 * (warp & 1), ti.bh);
            }
          } else {
            const int row0 = ti.pair * 128 + (warp & 3) * 32;
            if (row0 < p.n_pad) tma_store_3d(&tmO, stg, cc * 32, row0, ti.bh);
          }
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(o_free);                        // O_0/O_1 (and the far output) have been read
      if (p.lse && row_exists && wg == 0) {
        float val = 0.f;
        if (valid) val = (Lsum > 0.f) ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
        p.lse[(size_t)ti.bh * p.n_pad + tok] = val;
      }
      g += kPre + 2 * n_steps;
      J += n_steps;
      ++i;
    }
  }

  if (warp < 8 && lane == 0) bulk_wait_all();   // output stores complete
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
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = kp.n_tiles < sms ? kp.n_tiles : sms;
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kThreads, L::kBytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], kp);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap* maps, const AttnKParams& kp, cudaStream_t st) {
  if (a.tile3d) return a.gated ? launch_variant<D, true, true, false>(a, maps, kp, st)
                               : launch_variant<D, true, false, false>(a, maps, kp, st);
  if (a.Hs) return launch_variant<D, false, false, true>(a, maps, kp, st);
  return launch_variant<D, false, false, false>(a, maps, kp, st);
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  const int D = a.d;
  CUtensorMap maps[7];
  const uint64_t rowb = (uint64_t)D * 2;
  if (a.tile3d) {
    // Q (raster) by 4x4x4 tile boxes; K and V arrive in tile-major order, a tile = 64 rows
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)a.Ww, (uint64_t)a.Hh, (uint64_t)a.F, (uint64_t)a.BH};
    const uint64_t strides[4] = {rowb, rowb * a.Ww, rowb * a.Ww * a.Hh, rowb * a.Ww * a.Hh * a.F};
    const uint32_t box[5] = {64, 4, 4, 4, 1};
    if (!make_tile_map(&maps[0], a.q, 5, dims, strides, box)) return cudaErrorInvalidValue;
    const uint64_t kdims[3] = {(uint64_t)D, (uint64_t)a.s.n_pad, (uint64_t)a.BH};
    const uint64_t kstrides[2] = {rowb, rowb * a.s.n_pad};
    const uint32_t boxkv[3] = {64, 64, 1};
    if (!make_tile_map(&maps[1], a.k, 3, kdims, kstrides, boxkv)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[2], a.v, 3, kdims, kstrides, boxkv)) return cudaErrorInvalidValue;
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
  maps[5] = maps[0];
  if (a.tile3d) {
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)a.Ww, (uint64_t)a.Hh, (uint64_t)a.F, (uint64_t)a.BH};
    const uint64_t strides[4] = {rowb, rowb * a.Ww, rowb * a.Ww * a.Hh, rowb * a.Ww * a.Hh * a.F};
    const uint32_t boxo[5] = {32, 4, 4, 2, 1};
    if (!make_tile_map(&maps[6], a.out, 5, dims, strides, boxo, 64)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.s.n_pad, (uint64_t)a.BH};
    const uint64_t strides[2] = {rowb, rowb * a.s.n_pad};
    const uint32_t boxo[3] = {32, 32, 1};
    if (!make_tile_map(&maps[6], a.out, 3, dims, strides, boxo, 64)) return cudaErrorInvalidValue;
  }
  if (a.gated) {
    const uint64_t dims[3] = {(uint64_t)D, 64, (uint64_t)a.BH};
    const uint64_t strides[2] = {rowb, rowb * 64};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tile_map(&maps[3], a.kf, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[4], a.vf, 3, dims, strides, box)) return cudaErrorInvalidValue;
  } else if (a.Hs) {
    // [H'^T ; Z] rows of each query block: the D rows of H'^T, and the Z row
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(D + 1), (uint64_t)a.BH * a.n_qb};
    const uint64_t strides[2] = {rowb, rowb * (D + 1)};
    const uint32_t boxh[3] = {64, (uint32_t)D, 1};
    const uint32_t boxz[3] = {64, 1, 1};
    if (!make_tile_map(&maps[3], a.Hs, 3, dims, strides, boxh)) return cudaErrorInvalidValue;
    if (!make_tile_map(&maps[4], a.Hs, 3, dims, strides, boxz, 0)) return cudaErrorInvalidValue;   // read as a plain row
    if (!a.phi_q) return cudaErrorInvalidValue;
    const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)a.s.n_pad, (uint64_t)a.BH};
    const uint64_t qstrides[2] = {rowb, rowb * a.s.n_pad};
    const uint32_t boxq[3] = {64, 128, 1};
    if (!make_tile_map(&maps[5], a.phi_q, 3, qdims, qstrides, boxq)) return cudaErrorInvalidValue;
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
  kp.n_tiles = a.n_pairs * a.BH;
  kp.tile_counter = a.tile_counter;
  if (!a.tile_counter) return cudaErrorInvalidValue;
  if (cudaMemsetAsync(a.tile_counter, 0, sizeof(int), st) != cudaSuccess) return cudaErrorInvalidValue;
  return D == 128 ? launch_d<128>(a, maps, kp, st) : launch_d<64>(a, maps, kp, st);
}

}  // namespace slr
