// Definitions shared by the two decode paths (decode.cu: clustered CUDA-core
// kernel for fp32 caches and wide GQA groups; decode_tc.cu: persistent
// tensor-core kernel for bf16 caches with up to 8 query heads per KV head).
#pragma once

#include "internal.h"

namespace kvc {

constexpr int kMaxG = 16;    // query heads per KV head accepted by kv_decode_attn_update
constexpr int kTcMaxG = 8;   // ... on the tensor-core path

// One decode step of every row: the step's inputs and the cache it updates.
struct DecArgs {
  RowMap map;
  int G, d, C, S_cap;  // C, S_cap: cluster size and slots per CTA of the clustered path
  float scale2;        // log2(e) / sqrt(d)
  float gamma;
  int T, recent_pct;
  const void* q;
  const void* k;
  const void* v;
  void* out;
  void* Kc;
  void* Vc;
  float* A;
  int32_t* pos;
  const int64_t* slot_off;
  const int32_t* b;
  int32_t* meta;
  int32_t* status;
};

// An eviction candidate.
struct Best {
  float A;
  int pos;
  int slot;
};
// smaller A wins; equal A: the larger position is evicted
__device__ __forceinline__ bool better(const Best& x, const Best& y) {
  return x.A < y.A || (x.A == y.A && x.pos > y.pos);
}

// Largest b_i + 1 a row of the batch can have.
int cap_bound_of(const kv_shape& sh, const RowMap& m, const kv_params& p);

// Tensor-core path (decode_tc.cu).
size_t tc_scratch_bytes(const kv_shape& sh, const RowMap& m, int capb, long long total_slots);
int launch_tc_init(const kv_shape& sh, const RowMap& m, int capb, long long total_slots, const kv_cache& c,
                   cudaStream_t st);
int launch_tc(const kv_shape& sh, const RowMap& m, int capb, long long total_slots, const DecArgs& a,
              const kv_cache& c, cudaStream_t st);

}  // namespace kvc
