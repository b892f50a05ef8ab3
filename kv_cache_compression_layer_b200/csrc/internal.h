// Host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace kvc {

// Builds the row map of a batch; returns KV_OK or an error status.
int make_row_map(const kv_shape& sh, const int32_t* L, int32_t n_seq, RowMap& m);
int64_t total_keys(const RowMap& m);
int sm_count();
// 2-D bf16 tensor map over [rows][d] with a box of 64 x box_rows, 128-byte swizzle.
bool encode_rows_bf16(CUtensorMap* map, const void* base, int d, long long rows, int box_rows);

// Workspace layout of kv_score.
struct ScoreWs {
  size_t status_off;   // int32 status word
  size_t partial_off;  // float2 [total_tiles][R]
  size_t lse_off;      // float [rows][R]
  size_t bytes;
};
ScoreWs score_ws_layout(const RowMap& m, int R);

int launch_score(const kv_shape& sh, const RowMap& m, const void* qwin, const void* K, float* s, void* ws,
                 cudaStream_t st);
int launch_sss(const RowMap& m, const float* s, float* s_hat, int32_t* kstar, float alpha, float rho,
               cudaStream_t st);
int launch_allocate(const kv_shape& sh, const RowMap& m, const kv_params& p, const float* S, int32_t* b,
                    int64_t* slot_off, bool global, cudaStream_t st);
int launch_select_gather(const kv_shape& sh, const RowMap& m, const float* s_hat, const void* K, const void* V,
                         const int32_t* b, const int64_t* slot_off, int32_t* idx, void* Kc, void* Vc, int nseg,
                         cudaStream_t st);
constexpr int kMaxSelectSegments = 4096;
size_t decode_scratch_bytes(const kv_shape& sh, const RowMap& m, const kv_params& p, long long total_slots);
int launch_decode_init(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c,
                       cudaStream_t st);
int launch_decode(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c, const void* q_t,
                  const void* k_t, const void* v_t, void* out, cudaStream_t st);

// Bounded device waits give up after this long by default (a safety net;
// never reached by a correct run); kv_set_wait_limit_ns changes it for later
// launches, and wait_limit_ns() is the value a launch passes to its kernels.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
unsigned long long wait_limit_ns();

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? KV_OK : KV_ERR_CUDA; }

}  // namespace kvc
