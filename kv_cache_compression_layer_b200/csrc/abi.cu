// extern "C" entry points of libkvcomp.so: argument checks, row maps and
// workspace layout on the host, then the kernel launches. Declarations and
// argument documentation are in include/kvcomp.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace kvc {

static bool factors_ok(int n) {
  for (int p : {2, 3, 5, 7})
    while (n % p == 0) n /= p;
  return n == 1;
}

static bool shape_ok(const kv_shape* sh) {
  if (!sh) return false;
  if (sh->n_layers < 1 || sh->n_kv_heads < 1 || sh->n_kv_heads > 1024 || sh->group < 1) return false;
  if (sh->head_dim != 64 && sh->head_dim != 128) return false;
  if (sh->w < 0 || sh->group * sh->w > 256 || sh->group * sh->w < 1) return false;
  if (sh->dtype != KV_BF16 && sh->dtype != KV_F32) return false;
  return true;
}

int make_row_map(const kv_shape& sh, const int32_t* L, int32_t n_seq, RowMap& m) {
  if (!L || n_seq < 1 || n_seq > KV_MAX_SEQ) return KV_ERR_ARG;
  std::memset(&m, 0, sizeof(m));
  m.n_seq = n_seq;
  m.rows_per_seq = sh.n_layers * sh.n_kv_heads;
  m.n_rows = n_seq * m.rows_per_seq;
  long long key = 0;
  int tiles = 0;
  for (int s = 0; s < n_seq; ++s) {
    const int l = L[s];
    if (l < 2 || l % 2 || l > KV_MAX_L || l < sh.w || !factors_ok(l / 2)) return KV_ERR_UNSUPPORTED_L;
    m.L[s] = l;
    m.key_off[s] = key;
    m.tile_off[s] = tiles;
    key += (long long)m.rows_per_seq * l;
    tiles += m.rows_per_seq * ((l + kTileKeys - 1) / kTileKeys);
  }
  m.key_off[n_seq] = key;
  m.tile_off[n_seq] = tiles;
  return KV_OK;
}

int64_t total_keys(const RowMap& m) { return m.key_off[m.n_seq]; }

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_rows_bf16(CUtensorMap* map, const void* base, int d, long long rows, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static std::atomic<unsigned long long> g_wait_limit_ns{kWaitLimitNs};
unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

static bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Host-side fault injection for tests: KV_FAULT_INJECT=<entry point name>
// makes that entry point fail with KV_ERR_CUDA before launching anything.
static bool fault_injected(const char* name) {
  const char* v = std::getenv("KV_FAULT_INJECT");
  return v && std::strcmp(v, name) == 0;
}

// Readers of the kernel files' check words (debug builds register one per
// file while the library loads; release builds register none).
struct CheckReaders {
  int n = 0;
  int (*fn[32])(bool);
};
CheckReaders& check_readers() {
  static CheckReaders r;
  return r;
}
void register_check_word(int (*reader)(bool)) {
  CheckReaders& r = check_readers();
  if (r.n < 32) r.fn[r.n++] = reader;
}

}  // namespace kvc

using namespace kvc;

extern "C" {

int64_t kv_rows(const kv_shape* shape, int32_t n_seq) {
  if (!shape_ok(shape) || n_seq < 1 || n_seq > KV_MAX_SEQ) return -1;
  return (int64_t)n_seq * shape->n_layers * shape->n_kv_heads;
}

int kv_check_lengths(const kv_shape* shape, const int32_t* L, int32_t n_seq) {
  if (!shape_ok(shape)) return KV_ERR_ARG;
  RowMap m;
  return make_row_map(*shape, L, n_seq, m);
}

size_t kv_workspace_bytes(const kv_shape* shape, const int32_t* L, int32_t n_seq) {
  if (!shape_ok(shape)) return 0;
  RowMap m;
  if (make_row_map(*shape, L, n_seq, m) != KV_OK) return 0;
  return score_ws_layout(m, shape->group * shape->w).bytes;
}

int64_t kv_total_slots(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params) {
  if (!shape_ok(shape) || !params || !L || n_seq < 1 || n_seq > KV_MAX_SEQ) return -1;
  if (params->budget_pct < 1 || params->budget_pct > 100) return -1;
  int64_t total = 0;
  const int64_t H = shape->n_kv_heads;
  for (int s = 0; s < n_seq; ++s) {
    const int64_t B = ((int64_t)params->budget_pct * L[s] * H) / 100;
    total += (int64_t)shape->n_layers * (B + H);
  }
  return total;
}

size_t kv_decode_scratch_bytes(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                               int64_t total_slots) {
  if (!shape_ok(shape) || !params) return 0;
  RowMap m;
  if (make_row_map(*shape, L, n_seq, m) != KV_OK) return 0;
  if (total_slots <= 0) total_slots = kv_total_slots(shape, L, n_seq, params);
  if (total_slots <= 0) return 0;
  return decode_scratch_bytes(*shape, m, *params, total_slots);
}

int kv_score(const kv_shape* shape, const int32_t* L, int32_t n_seq, const void* qwin, const void* K, float* s,
             void* ws, size_t ws_bytes, void* stream) {
  if (fault_injected("kv_score")) return KV_ERR_CUDA;
  if (!shape_ok(shape)) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  if (!aligned16(qwin) || !aligned16(K) || !aligned16(s)) return KV_ERR_ARG;
  if (!ws || ws_bytes < score_ws_layout(m, shape->group * shape->w).bytes || !aligned16(ws)) return KV_ERR_WORKSPACE;
  return launch_score(*shape, m, qwin, K, s, ws, static_cast<cudaStream_t>(stream));
}

int kv_sss(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s, float* s_hat, int32_t* kstar,
           float alpha, float rho, void* stream) {
  if (fault_injected("kv_sss")) return KV_ERR_CUDA;
  if (!shape_ok(shape)) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  if (!aligned16(s) || !aligned16(s_hat) || !aligned16(kstar) || s == s_hat) return KV_ERR_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f) || !(rho >= 0.f && rho <= 1.f)) return KV_ERR_ARG;
  return launch_sss(m, s, s_hat, kstar, alpha, rho, static_cast<cudaStream_t>(stream));
}

int kv_allocate(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params, const float* S,
                int32_t* b, int64_t* slot_off, void* stream) {
  if (fault_injected("kv_allocate")) return KV_ERR_CUDA;
  if (!shape_ok(shape) || !params) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  if (!aligned16(S) || !aligned16(b) || !aligned16(slot_off)) return KV_ERR_ARG;
  if (params->budget_pct < 1 || params->budget_pct > 100 || !(params->r >= 0.f && params->r <= 1.f))
    return KV_ERR_ARG;
  for (int s = 0; s < n_seq; ++s) {
    const long long B = ((long long)params->budget_pct * L[s] * shape->n_kv_heads) / 100;
    if (B < (long long)shape->n_kv_heads * shape->w) return KV_ERR_BUDGET;
  }
  return launch_allocate(*shape, m, *params, S, b, slot_off, false, static_cast<cudaStream_t>(stream));
}

int kv_allocate_global(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                       const float* S, int32_t* b, int64_t* slot_off, void* stream) {
  if (fault_injected("kv_allocate_global")) return KV_ERR_CUDA;
  if (!shape_ok(shape) || !params) return KV_ERR_ARG;
  if ((long long)shape->n_layers * shape->n_kv_heads > 1024) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  if (!aligned16(S) || !aligned16(b) || !aligned16(slot_off)) return KV_ERR_ARG;
  if (params->budget_pct < 1 || params->budget_pct > 100 || !(params->r >= 0.f && params->r <= 1.f))
    return KV_ERR_ARG;
  for (int s = 0; s < n_seq; ++s) {
    const long long B = ((long long)params->budget_pct * L[s] * shape->n_kv_heads) / 100;
    if (B < (long long)shape->n_kv_heads * shape->w) return KV_ERR_BUDGET;
  }
  return launch_allocate(*shape, m, *params, S, b, slot_off, true, static_cast<cudaStream_t>(stream));
}

// The address a kernel reads a gather source at: device or managed memory as
// is, pinned host memory at its device mapping; nullptr for memory the device
// cannot read (pageable host memory).
static const void* gather_source(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return p;
  if (at.type == cudaMemoryTypeHost && at.devicePointer) return at.devicePointer;
  return nullptr;
}

int kv_select_gather(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s_hat, const void* K,
                     const void* V, const int32_t* b, const int64_t* slot_off, int32_t* idx, void* Kc, void* Vc,
                     void* stream) {
  if (fault_injected("kv_select_gather")) return KV_ERR_CUDA;
  if (!shape_ok(shape)) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  for (const void* p : {(const void*)s_hat, K, V, (const void*)b, (const void*)slot_off, (const void*)idx,
                        (const void*)Kc, (const void*)Vc})
    if (!aligned16(p)) return KV_ERR_ARG;
  K = gather_source(K);
  V = gather_source(V);
  if (!K || !V) return KV_ERR_ARG;
  return launch_select_gather(*shape, m, s_hat, K, V, b, slot_off, idx, Kc, Vc, 0, static_cast<cudaStream_t>(stream));
}

int kv_select_gather_segmented(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s_hat,
                               const void* K, const void* V, const int32_t* b, const int64_t* slot_off,
                               int32_t n_segments, int32_t* idx, void* Kc, void* Vc, void* stream) {
  if (fault_injected("kv_select_gather_segmented")) return KV_ERR_CUDA;
  if (!shape_ok(shape) || n_segments < 1 || n_segments > kMaxSelectSegments) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  for (const void* p : {(const void*)s_hat, K, V, (const void*)b, (const void*)slot_off, (const void*)idx,
                        (const void*)Kc, (const void*)Vc})
    if (!aligned16(p)) return KV_ERR_ARG;
  K = gather_source(K);
  V = gather_source(V);
  if (!K || !V) return KV_ERR_ARG;
  return launch_select_gather(*shape, m, s_hat, K, V, b, slot_off, idx, Kc, Vc, n_segments,
                              static_cast<cudaStream_t>(stream));
}

static bool cache_ok(const kv_cache* c) {
  return c && aligned16(c->Kc) && aligned16(c->Vc) && aligned16(c->A) && aligned16(c->pos) &&
         aligned16(c->slot_off) && aligned16(c->b) && aligned16(c->meta) && c->status;
}

static bool decode_params_ok(const kv_params* p) {
  return p && p->budget_pct >= 1 && p->budget_pct <= 100 && p->sinks_T >= 0 && p->recent_pct >= 0 &&
         p->recent_pct <= 100 && p->gamma >= 0.f && p->gamma <= 1.f;
}

int kv_decode_init(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                   kv_cache* cache, void* stream) {
  if (fault_injected("kv_decode_init")) return KV_ERR_CUDA;
  if (!shape_ok(shape) || !decode_params_ok(params) || !cache_ok(cache)) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  return launch_decode_init(*shape, m, *params, *cache, static_cast<cudaStream_t>(stream));
}

int kv_decode_attn_update(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                          kv_cache* cache, const void* q_t, const void* k_t, const void* v_t, void* out,
                          void* stream) {
  if (fault_injected("kv_decode_attn_update")) return KV_ERR_CUDA;
  if (!shape_ok(shape) || !decode_params_ok(params) || !cache_ok(cache)) return KV_ERR_ARG;
  RowMap m;
  int st = make_row_map(*shape, L, n_seq, m);
  if (st) return st;
  if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(out)) return KV_ERR_ARG;
  return launch_decode(*shape, m, *params, *cache, q_t, k_t, v_t, out, static_cast<cudaStream_t>(stream));
}

uint64_t kv_set_wait_limit_ns(uint64_t limit_ns) {
  return g_wait_limit_ns.exchange(limit_ns, std::memory_order_relaxed);
}

int kv_read_device_status(const int32_t* status_dev, int32_t* status_host, void* stream) {
  if (!status_dev || !status_host) return KV_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status_host, status_dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KV_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

int kv_debug_checks(void) {
#ifdef KV_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

int kv_debug_check_word(int32_t* word_host, int32_t clear) {
  if (!word_host) return KV_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return KV_ERR_CUDA;
  int w = 0;
  for (int i = 0; i < kvc::check_readers().n; ++i) {
    const int v = kvc::check_readers().fn[i](clear != 0);
    if (v < 0) return KV_ERR_CUDA;
    w |= v;
  }
  *word_host = w;
  return KV_OK;
}

const char* kv_status_string(int status) {
  switch (status) {
    case KV_OK: return "ok";
    case KV_ERR_ARG: return "invalid argument";
    case KV_ERR_UNSUPPORTED_L: return "unsupported audio length";
    case KV_ERR_BUDGET: return "budget too small";
    case KV_ERR_WORKSPACE: return "workspace missing or too small";
    case KV_ERR_CUDA: return "CUDA error";
    case KV_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
