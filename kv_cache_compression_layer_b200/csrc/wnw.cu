// kv_wnw_update / kv_wnw_recall: WnW's anchor-chunk importance with top-k
// selection and release hysteresis, and the recall of the tidal heads'
// chunks from host memory ("WnW: Waxing-and-Waning KV Cache for Long-Form
// Speech LLMs", 方法概述和架构 and 细节详述).
//
// score kernel (a CTA per 32 chunks of a sequence): stages the anchor rows'
// span of its chunks in shared memory with coalesced loads; each thread sums
// its chunk in float64 in a fixed order (anchor rows outer, the chunk's rows
// inner), so the selection does not depend on the thread layout.
//
// update kernel (one CTA per sequence): the sequence's scores and state are
// staged in shared memory when they fit; top_c rounds of a block argmax pick
// the chunks; the idle counts follow; releases, free slots and fetches are
// compacted in ascending order by block scans; the state is written back.
//
// recall kernel (persistent): a warp copies one fetched block of one tidal
// row, K or V, from the pinned host copy with 16-byte loads (four in flight
// per lane) into its slot of the GPU copy.
#include <algorithm>
#include <cstring>

#include "../../include/kvcomp_next.h"
#include "internal.h"

namespace kvc {
namespace {

struct WnwMap {
  int n_seq;
  int L[KV_MAX_SEQ];
  int M[KV_MAX_SEQ];
  int nb[KV_MAX_SEQ];
  long long s_off[KV_MAX_SEQ + 1];      // first anchor value (update) or host row (recall) of sequence s
  long long score_off[KV_MAX_SEQ + 1];  // first chunk score
  long long state_off[KV_MAX_SEQ + 1];  // first state word
};

bool params_ok(const kv_wnw_params* p) {
  if (!p) return false;
  const int C = p->chunk_len, S = p->chunk_stride;
  if (S < 1 || C < S || C % S || C > KV_WNW_MAX_CHUNK) return false;
  if (p->top_c < 1 || p->top_c > KV_WNW_MAX_TOP || p->release_after < 1) return false;
  const long long need = (long long)p->top_c * p->release_after * (C / S);
  return p->n_slots >= need && p->n_slots <= KV_WNW_MAX_SLOTS;
}

// Row layout of a batch; rows_per_seq anchor (or tidal) rows of L[s] each.
int wnw_layout(const int32_t* L, int n_seq, const kv_wnw_params* p, long long rows_per_seq, WnwMap& m) {
  if (!L || n_seq < 1 || n_seq > KV_MAX_SEQ || !params_ok(p)) return KV_ERR_ARG;
  std::memset(&m, 0, sizeof(m));
  m.n_seq = n_seq;
  const int C = p->chunk_len, S = p->chunk_stride;
  long long so = 0, sc = 0, st = 0;
  for (int s = 0; s < n_seq; ++s) {
    const int l = L[s];
    if (l < 1 || l > KV_WNW_MAX_L) return KV_ERR_ARG;
    m.L[s] = l;
    m.M[s] = l <= C ? 1 : (l - C + S - 1) / S + 1;
    m.nb[s] = (l + S - 1) / S;
    m.s_off[s] = so;
    m.score_off[s] = sc;
    m.state_off[s] = st;
    so += rows_per_seq * l;
    sc += m.M[s];
    st += (long long)m.M[s] + m.nb[s] + p->n_slots;
  }
  m.s_off[n_seq] = so;
  m.score_off[n_seq] = sc;
  m.state_off[n_seq] = st;
  return KV_OK;
}

constexpr int kScoreThreads = 128;
constexpr int kScoreChunks = 32;    // chunks per score CTA, at most
constexpr int kStageFloats = 24576; // anchor-row floats staged per round (96 KB)
static_assert(KV_WNW_MAX_CHUNK < kStageFloats, "a chunk fits the staged rows");

// Chunks per score CTA: at most kScoreChunks, and their span of rows fits the stage.
int chunks_per_cta(int C, int S) { return std::min(kScoreChunks, (kStageFloats - C) / S + 1); }

// Each round stages the span of the CTA's chunks for as many anchor rows as
// fit (coalesced loads, one round trip), then every thread adds its chunk's
// rows of those anchors to its float64 sum, anchors in order.
__global__ void __launch_bounds__(kScoreThreads)
    wnw_score_kernel(const WnwMap m, int C, int S, int cpc, int n_anchor, const float* __restrict__ s,
                     double* __restrict__ score) {
  extern __shared__ float stage[];  // [kStageFloats]
  const int sq = blockIdx.y;
  const int M = m.M[sq], L = m.L[sq];
  const int c0 = blockIdx.x * cpc;
  if (c0 >= M) return;  // the whole CTA
  const int c1 = min(M, c0 + cpc);
  const int p0 = c0 * S, plen = min(L, (c1 - 1) * S + C) - p0;
  const int na = max(1, kStageFloats / plen);  // anchor rows per round
  const int c = c0 + (int)threadIdx.x;
  const bool mine = c < c1;
  const int lo = c * S - p0, hi = min(c * S + C, L) - p0;
  const float* rows = s + m.s_off[sq] + p0;
  double acc = 0.0;
  for (int a0 = 0; a0 < n_anchor; a0 += na) {
    const int nr = min(na, n_anchor - a0);
    __syncthreads();  // the previous round's rows are consumed
    for (int i = threadIdx.x; i < nr * plen; i += kScoreThreads) {
      const int a = i / plen, j = i - a * plen;
      stage[i] = __ldg(rows + (long long)(a0 + a) * L + j);
    }
    __syncthreads();
    if (mine)
      for (int a = 0; a < nr; ++a)
        for (int j = lo; j < hi; ++j) acc = __dadd_rn(acc, (double)stage[a * plen + j]);
  }
  if (mine) score[m.score_off[sq] + c] = acc;
}

constexpr int kUpdThreads = 1024;
constexpr int kUpdStageMax = 200 * 1024;  // dynamic shared memory of the update kernel, at most
constexpr int kUpdWarps = kUpdThreads / 32;

// Exclusive sum over the block in thread order; *total = the block's sum.
__device__ int block_excl_sum(int v, int* total, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kUpdWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh[32 + lane] = w;
  }
  __syncthreads();
  const int before = (warp ? sh[32 + warp - 1] : 0) + x - v;
  *total = sh[32 + kUpdWarps - 1];
  __syncthreads();  // sh is free for the next call
  return before;
}

// (larger score, then lower chunk) wins; i < 0 is "none"
__device__ __forceinline__ bool beats(double v, int i, double bv, int bi) {
  return i >= 0 && (bi < 0 || v > bv || (v == bv && i < bi));
}

__device__ void block_argmax(double& v, int& i, double* shv, int* shi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_down_sync(0xffffffffu, v, o);
    const int oi = __shfl_down_sync(0xffffffffu, i, o);
    if (beats(ov, oi, v, i)) {
      v = ov;
      i = oi;
    }
  }
  if (lane == 0) {
    shv[warp] = v;
    shi[warp] = i;
  }
  __syncthreads();
  if (warp == 0) {
    v = lane < kUpdWarps ? shv[lane] : 0.0;
    i = lane < kUpdWarps ? shi[lane] : -1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_down_sync(0xffffffffu, v, o);
      const int oi = __shfl_down_sync(0xffffffffu, i, o);
      if (beats(ov, oi, v, i)) {
        v = ov;
        i = oi;
      }
    }
    if (lane == 0) {
      shv[0] = v;
      shi[0] = i;
    }
  }
  __syncthreads();
  v = shv[0];
  i = shi[0];
  __syncthreads();
}

// Is block b held by a resident chunk (chunks b - q + 1 .. b)?
__device__ __forceinline__ bool held(const int32_t* idle, int b, int q, int M) {
  for (int c = max(0, b - q + 1); c <= min(b, M - 1); ++c)
    if (idle[c] >= 0) return true;
  return false;
}

__global__ void __launch_bounds__(kUpdThreads)
    wnw_update_kernel(const WnwMap m, int C, int S, int top_c, int R, int n_slots, int cap, int staged,
                      int32_t* __restrict__ state, const double* __restrict__ score,
                      int32_t* __restrict__ fetch, int32_t* __restrict__ release, int32_t* __restrict__ counts) {
  // dynamic shared memory: free_list [n_slots]; when staged, the sequence's
  // scores [M] (8-byte aligned) and state words [M + nb + n_slots] after it
  extern __shared__ __align__(8) int dyn[];
  int* free_list = dyn;
  __shared__ int sh[64];
  __shared__ double shv[kUpdWarps];
  __shared__ int shi[kUpdWarps];
  __shared__ int sel[KV_WNW_MAX_TOP];
  const int q = C / S;
  const int sq = blockIdx.x;
  const int M = m.M[sq], nb = m.nb[sq];
  const double* sc = score + m.score_off[sq];
  int32_t* const g_state = state + m.state_off[sq];
  const int words = M + nb + n_slots;
  int32_t* idle = g_state;
  if (staged) {  // every phase below then works on shared memory
    double* sc_s = reinterpret_cast<double*>(dyn + ((n_slots + 1) & ~1));
    int32_t* st_s = reinterpret_cast<int32_t*>(sc_s + M);
    for (int i = threadIdx.x; i < M; i += kUpdThreads) sc_s[i] = sc[i];
    for (int i = threadIdx.x; i < words; i += kUpdThreads) st_s[i] = g_state[i];
    __syncthreads();
    sc = sc_s;
    idle = st_s;
  }
  int32_t* block_slot = idle + M;
  int32_t* slot_block = block_slot + nb;
  int32_t* fl = fetch + (long long)sq * cap * 2;
  int32_t* rl = release + (long long)sq * cap * 2;

  // 2. top_c chunks (the scores come from wnw_score_kernel), one block argmax per pick
  const int n_sel = min(top_c, M);
  for (int k = 0; k < n_sel; ++k) {
    double bv = 0.0;
    int bi = -1;
    for (int c = threadIdx.x; c < M; c += kUpdThreads) {
      bool taken = false;
      for (int t = 0; t < k; ++t) taken |= sel[t] == c;
      if (!taken && beats(sc[c], c, bv, bi)) {
        bv = sc[c];
        bi = c;
      }
    }
    block_argmax(bv, bi, shv, shi);
    if (threadIdx.x == 0) sel[k] = bi;
    __syncthreads();
  }

  // 3. idle counts
  for (int c = threadIdx.x; c < M; c += kUpdThreads) {
    bool chosen = false;
    for (int t = 0; t < n_sel; ++t) chosen |= sel[t] == c;
    int v = idle[c];
    if (chosen) {
      v = 0;
    } else if (v >= 0) {
      v += 1;
      if (v >= R) v = -1;
    }
    idle[c] = v;
  }
  __syncthreads();

  // 4. releases, ascending block order
  int carry = 0;
  for (int base = 0; base < nb; base += kUpdThreads) {
    const int b = base + threadIdx.x;
    int slot = -1;
    bool rel = false;
    if (b < nb) {
      slot = block_slot[b];
      rel = slot >= 0 && slot < n_slots && !held(idle, b, q, M);  // a slot past n_slots is never written
    }
    int tot;
    const int r = carry + block_excl_sum(rel ? 1 : 0, &tot, sh);
    if (rel) {
      if (r < cap) {
        rl[2 * r] = b;
        rl[2 * r + 1] = slot;
      }
      slot_block[slot] = -1;
      block_slot[b] = -1;
    }
    carry += tot;
  }
  const int n_rel = carry;
  __syncthreads();

  // 5. free slots, lowest first
  carry = 0;
  for (int base = 0; base < n_slots; base += kUpdThreads) {
    const int k = base + threadIdx.x;
    const bool f = k < n_slots && slot_block[k] < 0;
    int tot;
    const int r = carry + block_excl_sum(f ? 1 : 0, &tot, sh);
    if (f) free_list[r] = k;
    carry += tot;
  }
  const int n_free = carry;
  __syncthreads();

  // 6. fetches: the new blocks, ascending, take the free slots in order
  carry = 0;
  for (int base = 0; base < nb; base += kUpdThreads) {
    const int b = base + threadIdx.x;
    const bool nw = b < nb && block_slot[b] < 0 && held(idle, b, q, M);
    int tot;
    const int r = carry + block_excl_sum(nw ? 1 : 0, &tot, sh);
    if (nw && r < n_free) {
      const int slot = free_list[r];
      block_slot[b] = slot;
      slot_block[slot] = b;
      if (r < cap) {
        fl[2 * r] = b;
        fl[2 * r + 1] = slot;
      }
    }
    carry += tot;
  }
  if (threadIdx.x == 0) {
    counts[2 * sq] = min(min(carry, n_free), cap);
    counts[2 * sq + 1] = min(n_rel, cap);
  }
  if (staged) {
    __syncthreads();
    for (int i = threadIdx.x; i < words; i += kUpdThreads) g_state[i] = idle[i];
  }
}

constexpr int kRecThreads = 256;

__global__ void __launch_bounds__(kRecThreads)
    wnw_recall_kernel(const WnwMap m, int S, int n_slots, int n_tidal, int row_bytes, int cap, long long units,
                      const int32_t* __restrict__ fetch, const int32_t* __restrict__ counts,
                      const uint8_t* __restrict__ K_host, const uint8_t* __restrict__ V_host,
                      uint8_t* __restrict__ K_gpu, uint8_t* __restrict__ V_gpu) {
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * kRecThreads) >> 5;
  for (long long u = ((long long)blockIdx.x * kRecThreads + threadIdx.x) >> 5; u < units; u += nw) {
    // u = ((sq * cap + f) * n_tidal + r) * 2 + (0: K, 1: V)
    const int kv = (int)(u & 1);
    long long t = u >> 1;
    const int r = (int)(t % n_tidal);
    t /= n_tidal;
    const int f = (int)(t % cap);
    const int sq = (int)(t / cap);
    if (f >= __ldg(counts + 2 * sq)) continue;
    const int b = __ldg(fetch + ((long long)sq * cap + f) * 2), slot = __ldg(fetch + ((long long)sq * cap + f) * 2 + 1);
    const int L = m.L[sq];
    const long long row0 = (long long)b * S;
    if (!kv_check(b >= 0 && row0 < L && slot >= 0 && slot < n_slots)) continue;
    const int rows = (int)min((long long)S, L - row0);
    const uint4* src = reinterpret_cast<const uint4*>((kv ? V_host : K_host) +
                                                      (m.s_off[sq] + (long long)r * L + row0) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>((kv ? V_gpu : K_gpu) +
                                          ((((long long)sq * n_tidal + r) * n_slots + slot) * S) * row_bytes);
    const int n16 = rows * (row_bytes / 16);
    for (int i = lane; i < n16; i += 128) {
      uint4 x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (i + 32 * k < n16) x[k] = src[i + 32 * k];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (i + 32 * k < n16) dst[i + 32 * k] = x[k];
    }
  }
}

// The device address of pinned host memory, or nullptr when p is not pinned host memory.
const void* host_device_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
  return at.devicePointer;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" {

int64_t kv_wnw_chunk_count(const int32_t* L, int32_t n_seq, const kv_wnw_params* p) {
  WnwMap m;
  if (wnw_layout(L, n_seq, p, 1, m) != KV_OK) return -1;
  return m.score_off[n_seq];
}

int64_t kv_wnw_state_ints(const int32_t* L, int32_t n_seq, const kv_wnw_params* p) {
  WnwMap m;
  if (wnw_layout(L, n_seq, p, 1, m) != KV_OK) return -1;
  return m.state_off[n_seq];
}

int kv_wnw_init(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t* state, void* stream) {
  WnwMap m;
  const int st = wnw_layout(L, n_seq, p, 1, m);
  if (st != KV_OK) return st;
  if (!state || (reinterpret_cast<uintptr_t>(state) & 3u)) return KV_ERR_ARG;
  return cuda_status(cudaMemsetAsync(state, 0xff, sizeof(int32_t) * (size_t)m.state_off[n_seq],
                                     static_cast<cudaStream_t>(stream)));
}

int kv_wnw_update(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t n_anchor, const float* s,
                  int32_t* state, double* score, int32_t* fetch, int32_t* release, int32_t* counts, void* stream) {
  if (n_anchor < 1 || n_anchor > 1024) return KV_ERR_ARG;
  WnwMap m;
  const int st = wnw_layout(L, n_seq, p, n_anchor, m);
  if (st != KV_OK) return st;
  if (!s || !state || !score || !fetch || !release || !counts) return KV_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(s) & 3u) || (reinterpret_cast<uintptr_t>(state) & 3u) ||
      (reinterpret_cast<uintptr_t>(score) & 7u) || (reinterpret_cast<uintptr_t>(fetch) & 3u) ||
      (reinterpret_cast<uintptr_t>(release) & 3u) || (reinterpret_cast<uintptr_t>(counts) & 3u))
    return KV_ERR_ARG;
  const int cap = p->top_c * (p->chunk_len / p->chunk_stride);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int cpc = chunks_per_cta(p->chunk_len, p->chunk_stride);
  int max_M = 0;
  for (int i = 0; i < n_seq; ++i) max_M = std::max(max_M, m.M[i]);
  // per-device settings: made on every launch (cheap), for whichever device is current
  if (cudaFuncSetAttribute(wnw_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(sizeof(float) * kStageFloats)) != cudaSuccess)
    return KV_ERR_CUDA;
  wnw_score_kernel<<<dim3((max_M + cpc - 1) / cpc, n_seq), kScoreThreads, sizeof(float) * kStageFloats, cs>>>(
      m, p->chunk_len, p->chunk_stride, cpc, n_anchor, s, score);
  // stage each sequence's scores and state in shared memory when the largest fits
  size_t stage_bytes = 0;
  for (int i = 0; i < n_seq; ++i)
    stage_bytes = std::max(stage_bytes, sizeof(double) * m.M[i] + sizeof(int32_t) * (m.M[i] + m.nb[i] + p->n_slots));
  const size_t list_bytes = sizeof(int32_t) * (size_t)((p->n_slots + 1) & ~1);
  const int staged = list_bytes + stage_bytes <= (size_t)kUpdStageMax ? 1 : 0;
  if (cudaFuncSetAttribute(wnw_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUpdStageMax) !=
      cudaSuccess)
    return KV_ERR_CUDA;
  wnw_update_kernel<<<n_seq, kUpdThreads, staged ? list_bytes + stage_bytes : list_bytes, cs>>>(
      m, p->chunk_len, p->chunk_stride, p->top_c, p->release_after, p->n_slots, cap, staged, state, score, fetch,
      release, counts);
  return cuda_status(cudaGetLastError());
}

int kv_wnw_recall(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t n_tidal, int32_t d, int32_t dtype,
                  const int32_t* fetch, const int32_t* counts, const void* K_host, const void* V_host, void* K_gpu,
                  void* V_gpu, void* stream) {
  if (n_tidal < 1 || (dtype != KV_BF16 && dtype != KV_F32)) return KV_ERR_ARG;
  const int esz = dtype == KV_BF16 ? 2 : 4;
  if (d < 1 || d > 16384 || (d * esz) % 16) return KV_ERR_ARG;
  WnwMap m;
  const int st = wnw_layout(L, n_seq, p, n_tidal, m);
  if (st != KV_OK) return st;
  if (!fetch || !counts || !K_host || !V_host || !K_gpu || !V_gpu) return KV_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(K_gpu) & 15u) || (reinterpret_cast<uintptr_t>(V_gpu) & 15u) ||
      (reinterpret_cast<uintptr_t>(K_host) & 15u) || (reinterpret_cast<uintptr_t>(V_host) & 15u))
    return KV_ERR_ARG;
  const void* kd = host_device_ptr(K_host);
  const void* vd = host_device_ptr(V_host);
  if (!kd || !vd) return KV_ERR_ARG;
  const int cap = p->top_c * (p->chunk_len / p->chunk_stride);
  const long long units = (long long)n_seq * cap * n_tidal * 2;
  const long long want = (units * 32 + kRecThreads - 1) / kRecThreads;
  const int grid = (int)std::max(1ll, std::min<long long>(want, (long long)sm_count() * 8));
  wnw_recall_kernel<<<grid, kRecThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      m, p->chunk_stride, p->n_slots, n_tidal, d * esz, cap, units, fetch, counts,
      static_cast<const uint8_t*>(kd), static_cast<const uint8_t*>(vd), static_cast<uint8_t*>(K_gpu),
      static_cast<uint8_t*>(V_gpu));
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
