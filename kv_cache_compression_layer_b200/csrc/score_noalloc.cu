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
#include "internal.h"

namespace kvc {
namespace {

static __device__ __align__(256) unsigned char g_score_scratch[KV_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device. In host code the
// array's name is only a stand-in, never a device address, so it is looked up
// on every call (a cheap host query): a cached address could outlive the
// module after a device reset.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || !p) return KV_ERR_CUDA;
  *out = p;
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

// The status word of the last kv_score_noalloc call on the current device
// sits at the start of the array (kv_score's workspace layout).
extern "C" int kv_score_noalloc_status(int32_t* status_host, void* stream) {
  if (!status_host) return KV_ERR_ARG;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != KV_OK) return st;
  return kv_read_device_status(static_cast<const int32_t*>(scratch), status_host, stream);
}
