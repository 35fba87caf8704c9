// Verify / resample / propose with no device allocation at all.
//
// isd_accept_propose needs a few hundred kilobytes of device scratch (the
// per-chunk vocabulary statistics) that its caller allocates. Some callers
// cannot allocate device memory: code running inside a host program that
// owns every byte of the GPU through its own fixed pool, code that must not
// enter the CUDA allocator once serving has started (an allocation can block
// or fail under memory pressure), or a plugin loaded into a process where it
// has no allocator of its own. isd_accept_propose_noalloc runs the same
// kernels with their scratch in a fixed array compiled into this library.
//
// The array below lives in device memory of every GPU that loads the library
// and stays there until the process exits. Its address is looked up once per
// device (cudaGetSymbolAddress, with that device current) on the first call
// made while that device is current; host code must not use the symbol's
// name as a pointer, since in host code it only stands in for the device
// object. With lazy module loading (CUDA's default) that first lookup also
// loads this translation unit's module onto the device, which places the
// array: the first call on a device allocates and can fail when the device
// is full, so callers make it at start-up; later calls allocate nothing.
// Every call shares the array, so calls whose work overlaps on the
// GPU (different streams, or devices sharing nothing but this library) race
// on it; callers must serialise them. The kernels write every scratch entry
// before they read it, so nothing needs clearing between calls.
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = 4u << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_accept_scratch[kScratchBytes];

void* g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_accept_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return isd::set_error(ISD_E_CUDA, (std::string("cudaGetDevice: ") + cudaGetErrorString(e)).c_str());
  if (dev < 0 || dev >= kMaxDevices)
    return isd::set_error(ISD_E_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_accept_scratch);
    if (e != cudaSuccess || !p)
      return isd::set_error(
          ISD_E_CUDA, (std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e)).c_str());
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return ISD_OK;
}

}  // namespace

extern "C" int isd_accept_propose_noalloc(const float* logits_dev, const isd_batch* batch,
                                          const isd_kv* kv, int32_t page_size, int32_t vocab,
                                          int32_t* pending_dev, float* q_cache_dev,
                                          const float* uniforms_dev, int32_t* out_accepted_dev,
                                          int32_t* out_committed_dev, int32_t* status_dev,
                                          void* stream) {
  if (!logits_dev || !batch || !kv || !pending_dev || !uniforms_dev || !out_accepted_dev ||
      !status_dev || !batch->seq_len_dev || !batch->n_draft_dev || !kv->page_table_dev ||
      !kv->free_list_dev || !kv->free_head_dev)
    return isd::set_error(ISD_E_INVALID, "null argument");
  const int B = batch->batch, N = batch->stride_n;
  if (B < 1 || B > 1024 || N < 1 || N > 8)
    return isd::set_error(ISD_E_INVALID, "batch or stride_n out of range");
  if (vocab < 4 || vocab % 4 || vocab > 64 * 8192) return isd::set_error(ISD_E_UNSUPPORTED, "vocab");
  if (page_size < 1) return isd::set_error(ISD_E_INVALID, "page_size");
  if ((batch->flags & ISD_PROPOSE_SAMPLE) && N > 1 && !q_cache_dev)
    return isd::set_error(ISD_E_INVALID, "SAMPLE proposals need q_cache");
  const size_t need = isd::accept_workspace_bytes(B, N, vocab);
  if (need > kScratchBytes) {
    const std::string msg = "isd_accept_propose_noalloc: this batch needs " + std::to_string(need) +
                            " bytes of scratch but the fixed array holds " +
                            std::to_string(kScratchBytes) +
                            " (batch * (2N-1) * ceil(vocab/8192) * 16 bytes of chunk statistics"
                            " and 4 bytes per request); use isd_accept_propose";
    return isd::set_error(ISD_E_UNSUPPORTED, msg.c_str());
  }
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  isd::AcceptArgs a;
  a.logits = logits_dev;
  a.batch = B;
  a.stride_n = N;
  a.vocab = vocab;
  a.flags = batch->flags;
  a.page_size = page_size;
  a.pending = pending_dev;
  a.n_draft = batch->n_draft_dev;
  a.seq_len = batch->seq_len_dev;
  a.q_cache = q_cache_dev;
  a.uniforms = uniforms_dev;
  a.accepted = out_accepted_dev;
  a.committed = out_committed_dev;
  a.page_table = kv->page_table_dev;
  a.free_list = kv->free_list_dev;
  a.free_head = kv->free_head_dev;
  a.num_pages = kv->num_pages;
  a.max_pages_per_req = kv->max_pages_per_req;
  a.free_count = kv->free_count;
  a.status = status_dev;
  cudaError_t e = isd::launch_accept(a, scratch, static_cast<cudaStream_t>(stream), nullptr);
  if (e != cudaSuccess)
    return isd::set_error(ISD_E_CUDA, (std::string("launch: ") + cudaGetErrorString(e)).c_str());
  return ISD_OK;
}
