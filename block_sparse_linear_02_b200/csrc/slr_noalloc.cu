// slr_noalloc.cu -- slr_block_sparse_attn_noalloc: the block-sparse attention
// call for callers that cannot hand the library a scratch buffer.
//
// Some callers cannot allocate device memory on the library's behalf: a host
// application that owns the whole device-memory budget (an inference server
// that reserves the GPU's memory up front and forbids any further cudaMalloc),
// or a plug-in whose own interface only passes the input and output tensors.
// This entry point needs no workspace: its scratch (the device status word and
// the per-pair key-block lists) lives in one file-scope static device array of
// kNoallocScratchBytes, which every GPU that loads the library holds until the
// process exits.  The call itself allocates nothing.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "../../include/slr.h"
#include "launch.h"

namespace {

constexpr size_t kNoallocScratchBytes = 4u << 20;   // 4 MiB, SLR_NOALLOC_SCRATCH_BYTES in slr.h
constexpr size_t kStatusBytes = 256;

// Shared by every call on a device; holds the last call's lists until the next call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device.  The host-side symbol is only a stand-in; kernels must get this address.
slr_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SLR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SLR_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SLR_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

namespace slr {

// slr_check_status(NULL, stream): the status word the no-workspace call writes into
// word 0 of the static scratch when its caller passes no status pointer.  Synchronises
// the stream, reads the word on the current device and clears it.
int noalloc_check_status(void* stream) {
  void* base = nullptr;
  slr_status st = scratch_address(&base);
  if (st != SLR_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SLR_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SLR_ERR_CUDA;
  if (cudaMemset(base, 0, sizeof(int)) != cudaSuccess) return SLR_ERR_CUDA;
  return code == 0 ? SLR_OK : -code;
}

}  // namespace slr

extern "C" slr_status slr_block_sparse_attn_noalloc(const void* q, const void* k, const void* v,
                                                    const slr_seq* seq, const int32_t* kv_idx,
                                                    const int32_t* kv_cnt, int kv_max, void* o,
                                                    float* lse_opt, int* status_opt, void* stream) {
  using namespace slr;
  if (!seq) return SLR_ERR_ARG;
  if (seq->B < 1 || seq->H < 1 || seq->n_seg < 1 || seq->seg_len < 1 || seq->seg_stride < 1) return SLR_ERR_ARG;
  if (seq->d != 64 && seq->d != 128) return SLR_ERR_UNSUPPORTED;
  if (seq->block != kBlock || seq->seg_stride % kBlock != 0) return SLR_ERR_UNSUPPORTED;
  if (seq->seg_len > seq->seg_stride || seq->seg_len <= seq->seg_stride - kBlock) return SLR_ERR_UNSUPPORTED;
  const long long n_pad = (long long)seq->n_seg * seq->seg_stride;
  const long long bh = (long long)seq->B * seq->H;
  if (n_pad / kBlock > kMaxKeyBlocks || bh > 65535) return SLR_ERR_UNSUPPORTED;
  auto al = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al(q) || !al(k) || !al(v) || !al(o)) return SLR_ERR_ARG;
  if (status_opt && (reinterpret_cast<uintptr_t>(status_opt) & 3u)) return SLR_ERR_ARG;
  if (kv_idx && (!kv_cnt || kv_max < 1)) return SLR_ERR_ARG;

  const int nb = (int)(n_pad / kBlock), npairs = (nb + 1) / 2;
  const int cap = kv_idx ? (int)(2LL * kv_max < nb ? 2LL * kv_max : nb) : 0;
  const size_t list_bytes = kv_idx ? align256((size_t)bh * npairs * cap * sizeof(uint32_t)) : 0;
  const size_t cnt_bytes = kv_idx ? align256((size_t)bh * npairs * sizeof(int32_t)) : 0;
  if (kStatusBytes + list_bytes + cnt_bytes > kNoallocScratchBytes) return SLR_ERR_WORKSPACE;

  void* base = nullptr;
  slr_status st = scratch_address(&base);
  if (st != SLR_OK) return st;
  uint8_t* scratch = static_cast<uint8_t*>(base);
  int* status = status_opt ? status_opt : reinterpret_cast<int*>(scratch);
  uint32_t* list = reinterpret_cast<uint32_t*>(scratch + kStatusBytes);
  int32_t* list_cnt = reinterpret_cast<int32_t*>(scratch + kStatusBytes + list_bytes);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return SLR_ERR_CUDA;
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = o; a.lse = lse_opt; a.status = status;
  a.tile_counter = reinterpret_cast<int*>(scratch) + 1;   // inside the status area of the scratch
  a.BH = (int)bh; a.d = seq->d;
  a.s = SeqShape{(int)n_pad, seq->seg_len, seq->seg_stride, nb};
  a.n_qb = nb; a.n_kb = nb; a.n_pairs = npairs; a.gate = 1.f;
  if (kv_idx) {
    ListArgs la;
    memset(&la, 0, sizeof(la));
    la.mode = kListExplicit;
    la.n_qb = nb; la.n_kb = nb; la.n_pairs = npairs; la.cap = cap;
    la.kv_idx = kv_idx; la.kv_cnt = kv_cnt; la.kv_max = kv_max;
    la.s = a.s; la.list = list; la.list_cnt = list_cnt; la.status = status;
    if (launch_pair_lists(la, (int)bh, s) != cudaSuccess) return SLR_ERR_CUDA;
    a.list = list; a.list_cnt = list_cnt; a.list_cap = cap; a.list_per_head = 1;
  }
  if (launch_attention(a, s) != cudaSuccess) return SLR_ERR_CUDA;
  return SLR_OK;
}
