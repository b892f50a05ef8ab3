// kv_score_noalloc: kv_score for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain scratch memory at the
// moment they score a prompt: a serving runtime that reserves the whole GPU
// for its own pool up front (so a cudaMalloc would fail, or would fragment
// that pool), a plugin whose host process owns every allocation and only
// hands in input and output buffers, or a latency-critical loop that must not
// pay for cudaMalloc's implicit synchronisation. This variant takes only the
// inputs and the output; its scratch (the per-tile softmax partials, the
// per-row denominators and the device status word) lives in one file-scope
// device array below, sized for batches up to KV_NOALLOC_SCRATCH_BYTES of
// scratch, which every GPU that loads the library holds until the process
// exits.
#include <mutex>

#include "internal.h"

namespace kvc {
namespace {

static __device__ __align__(256) unsigned char g_score_scratch[KV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device address).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || !p) return KV_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return KV_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" int kv_score_noalloc(const kv_shape* shape, const int32_t* L, int32_t n_seq, const void* qwin,
                                const void* K, float* s, void* stream) {
  const int chk = kv_check_lengths(shape, L, n_seq);
  if (chk != KV_OK) return chk;
  if (kv_workspace_bytes(shape, L, n_seq) > KV_NOALLOC_SCRATCH_BYTES) return KV_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != KV_OK) return st;
  return kv_score(shape, L, n_seq, qwin, K, s, scratch, KV_NOALLOC_SCRATCH_BYTES, stream);
}
