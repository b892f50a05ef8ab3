// kv_decode_attn_update: one decode step of every (sequence, layer, KV head)
// row over its compacted, slot-stable cache (VoxZip, second stage:
// A^(t) = gamma [A^(t-1), 0] + softmax(q_t K_t^T / sqrt d), then keep the T
// sinks, the M most recent entries and the top-N of the middle by A).
//
// One launch covers every row. Each row is a thread-block cluster of C CTAs;
// CTA c owns slots [c S, c S + S) of the row's b + 1 slots. Within a step:
//   1. the CTA that owns the free slot writes k_t, v_t, pos there;
//   2. every CTA computes its slots' logits for the g query heads (kept in
//      shared memory), its local softmax max / sum and its partial p V;
//   3. cluster rank 0 combines the partials over distributed shared memory,
//      writes the attention output and publishes log2 of the denominators;
//   4. every CTA turns its stored probabilities into the exact softmax,
//      updates A <- gamma A + sum_g p_g (0 for the appended entry) and finds
//      its smallest middle A (ties: the larger position);
//   5. rank 0 picks the row's eviction and updates the row's meta data.
// Nothing leaves the chip between the phases; the waits are hardware
// cluster barriers, not spin loops.
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kMaxG = 16;

struct DecArgs {
  RowMap map;
  int G, d, C, S_cap;
  float scale2;  // log2(e) / sqrt(d)
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

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& y, float x) { y = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& y, float x) { y = __float2bfloat16_rn(x); }

struct Best {
  float A;
  int pos;
  int slot;
};
// smaller A wins; equal A: the larger position is evicted
__device__ __forceinline__ bool better(const Best& x, const Best& y) {
  return x.A < y.A || (x.A == y.A && x.pos > y.pos);
}

template <typename TIn>
__global__ void __launch_bounds__(kDecThreads) decode_simple_kernel(const DecArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / a.C;
  const int G = a.G, d = a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ float dsm[];
  float* xs = dsm;                       // [G][S_cap] logits, then exp2(x - m)
  float* q_s = xs + G * a.S_cap;         // [G][d]
  float* o_s = q_s + G * d;              // [G][d]
  __shared__ float red[kDecWarps][kMaxG];
  __shared__ float m_s[kMaxG], z_s[kMaxG], lse_s[kMaxG];
  __shared__ Best bw[kDecWarps];
  __shared__ Best best_s;

  const int L = row_len(a.map, row);
  const long long base = a.slot_off[row];
  const int cap = (int)(a.slot_off[row + 1] - base);
  const int bb = a.b[row];
  int32_t* meta = a.meta + (long long)row * 8;
  const int count = meta[0], next = meta[1], steps = meta[2], count0 = meta[4];
  const int n = count + 1;  // present slots [0, n) once the new token is in
  const int pos_new = L + steps;
  const int M = (a.recent_pct * bb) / 100;
  const int appended = steps + 1;
  const bool evict = n > bb;
  const int S = (cap + a.C - 1) / a.C;
  const int j0 = rank * S, j1 = min(j0 + S, n);
  const bool ok = S <= a.S_cap && count < cap && (!evict || bb >= a.T + M);
  const int cnt = ok ? max(0, j1 - j0) : 0;
  if (!ok && rank == 0 && tid == 0) atomicOr(a.status, S > a.S_cap ? KV_DEV_CAPACITY : KV_DEV_BUDGET);

  const TIn* qin = static_cast<const TIn*>(a.q) + (long long)row * G * d;
  const TIn* kin = static_cast<const TIn*>(a.k) + (long long)row * d;
  const TIn* vin = static_cast<const TIn*>(a.v) + (long long)row * d;
  TIn* Kc = static_cast<TIn*>(a.Kc) + base * d;
  TIn* Vc = static_cast<TIn*>(a.Vc) + base * d;
  float* A = a.A + base;
  int32_t* pos = a.pos + base;

  for (int i = tid; i < G * d; i += kDecThreads) {
    q_s[i] = to_f(qin[i]);
    o_s[i] = 0.f;
  }
  const bool own_new = ok && next >= j0 && next < j1;
  if (own_new) {
    for (int i = tid; i < d; i += kDecThreads) {
      Kc[(long long)next * d + i] = kin[i];
      Vc[(long long)next * d + i] = vin[i];
    }
    if (tid == 0) pos[next] = pos_new;
  }
  __syncthreads();

  // ---- logits and local max
  float mx[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) mx[g] = -INFINITY;
  if (ok) {
    for (int jl = tid; jl < cnt; jl += kDecThreads) {
      const int j = j0 + jl;
      const TIn* kr = j == next ? kin : Kc + (long long)j * d;
      float x[kMaxG];
#pragma unroll
      for (int g = 0; g < kMaxG; ++g) x[g] = 0.f;
      for (int c = 0; c < d; c += 8) {
        float kv[8];
        if constexpr (sizeof(TIn) == 2) {
          const uint4 raw = *reinterpret_cast<const uint4*>(kr + c);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            kv[2 * e] = f.x;
            kv[2 * e + 1] = f.y;
          }
        } else {
          const float4 r0 = *reinterpret_cast<const float4*>(kr + c);
          const float4 r1 = *reinterpret_cast<const float4*>(kr + c + 4);
          kv[0] = r0.x; kv[1] = r0.y; kv[2] = r0.z; kv[3] = r0.w;
          kv[4] = r1.x; kv[5] = r1.y; kv[6] = r1.z; kv[7] = r1.w;
        }
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) {
          if (g < G) {
            const float* qg = q_s + g * d + c;
#pragma unroll
            for (int e = 0; e < 8; ++e) x[g] = fmaf(qg[e], kv[e], x[g]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        if (g < G) {
          const float xv = x[g] * a.scale2;
          xs[g * a.S_cap + jl] = xv;
          mx[g] = fmaxf(mx[g], xv);
        }
    }
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    if (g < G) {
      float v = mx[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) red[warp][g] = v;
    }
  }
  __syncthreads();
  if (tid < G) {
    float v = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) v = fmaxf(v, red[w][tid]);
    m_s[tid] = v;
  }
  __syncthreads();

  // ---- exp2(x - m) in place, local sums
  float zs[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) zs[g] = 0.f;
  for (int jl = tid; jl < cnt; jl += kDecThreads) {
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < G) {
        const float p = ex2_approx(xs[g * a.S_cap + jl] - m_s[g]);
        xs[g * a.S_cap + jl] = p;
        zs[g] += p;
      }
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    if (g < G) {
      float v = zs[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][g] = v;
    }
  }
  __syncthreads();
  if (tid < G) {
    float v = 0.f;
    for (int w = 0; w < kDecWarps; ++w) v += red[w][tid];
    z_s[tid] = v;
  }

  // ---- partial p V: each warp takes every kDecWarps-th slot, lanes own columns
  {
    const int per = d / 32;  // columns per lane (2 or 4)
    float acc[kMaxG][4];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;
    for (int jl = warp; jl < cnt; jl += kDecWarps) {
      const int j = j0 + jl;
      const TIn* vr = (j == next ? vin : Vc + (long long)j * d) + lane * per;
      float vv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) vv[e] = e < per ? to_f(vr[e]) : 0.f;
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        if (g < G) {
          const float p = xs[g * a.S_cap + jl];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[g][e] = fmaf(p, vv[e], acc[g][e]);
        }
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < G)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < per) atomicAdd(&o_s[g * d + lane * per + e], acc[g][e]);
  }
  cluster.sync();

  // ---- rank 0: combine the C partials, write the output, publish lse2
  if (rank == 0) {
    if (tid < G) {
      float Mx = -INFINITY;
      for (int r = 0; r < a.C; ++r) Mx = fmaxf(Mx, *cluster.map_shared_rank(&m_s[tid], r));
      float Z = 0.f;
      for (int r = 0; r < a.C; ++r) {
        const float mr = *cluster.map_shared_rank(&m_s[tid], r);
        if (mr > -INFINITY) Z += *cluster.map_shared_rank(&z_s[tid], r) * exp2f(mr - Mx);
      }
      lse_s[tid] = Mx + log2f(Z);
    }
    __syncthreads();
    TIn* out = static_cast<TIn*>(a.out) + (long long)row * G * d;
    for (int i = tid; i < G * d; i += kDecThreads) {
      const int g = i / d;
      float o = 0.f;
      for (int r = 0; r < a.C; ++r) {
        const float mr = *cluster.map_shared_rank(&m_s[g], r);
        if (mr > -INFINITY) o += *cluster.map_shared_rank(&o_s[i], r) * exp2f(mr - lse_s[g]);
      }
      from_f(out[i], o);
    }
  }
  cluster.sync();

  // ---- exact probabilities, A update, local eviction candidate
  Best best{INFINITY, -1, -1};
  {
    float f[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      f[g] = 0.f;
      if (g < G && m_s[g] > -INFINITY) f[g] = exp2f(m_s[g] - *cluster.map_shared_rank(&lse_s[g], 0));
    }
    int pos_thr;
    if (appended >= M) pos_thr = pos_new - M + 1;
    else pos_thr = pos[max(0, count0 - (M - appended))];
    if (ok) {
      for (int jl = tid; jl < cnt; jl += kDecThreads) {
        const int j = j0 + jl;
        float psum = 0.f;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) psum = fmaf(xs[g * a.S_cap + jl], f[g], psum);
        const float Anew = (j == next ? 0.f : a.gamma * A[j]) + psum;
        A[j] = Anew;
        const int pj = j == next ? pos_new : pos[j];
        if (j >= a.T && pj < pos_thr) {
          const Best c{Anew, pj, j};
          if (better(c, best)) best = c;
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Best y;
    y.A = __shfl_xor_sync(0xffffffffu, best.A, o);
    y.pos = __shfl_xor_sync(0xffffffffu, best.pos, o);
    y.slot = __shfl_xor_sync(0xffffffffu, best.slot, o);
    if (better(y, best)) best = y;
  }
  if (lane == 0) bw[warp] = best;
  __syncthreads();
  if (tid == 0) {
    Best bst = bw[0];
    for (int w = 1; w < kDecWarps; ++w)
      if (better(bw[w], bst)) bst = bw[w];
    best_s = bst;
  }
  cluster.sync();

  if (rank == 0 && tid == 0 && ok) {
    Best bst = best_s;
    for (int r = 1; r < a.C; ++r) {
      const Best y = *cluster.map_shared_rank(&best_s, r);
      if (better(y, bst)) bst = y;
    }
    if (evict && bst.slot >= 0) {
      meta[0] = bb;
      meta[1] = bst.slot;
      meta[3] = bst.slot;
    } else {
      meta[0] = n;
      meta[1] = n;
      meta[3] = -1;
    }
    meta[2] = steps + 1;
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
}


// ------------------------------------------------------------------------
// bf16 caches: persistent split-K tensor-core decode, then a per-row finish.
//
// decode_attn_kernel: every row is cut into work items of kCH slots; one CTA
// per SM takes a contiguous run of items. Its producer warp streams each
// item's 64-slot tiles of K and V, with the row's g query rows and a small
// header (row, slot range, the row's step state), through a 5-stage TMA ring
// (128-byte swizzled boxes, so the ldmatrix reads are free of bank
// conflicts). Eight consumer warps in two groups take alternate tiles; in a
// group each warp owns 16 slots of a tile and runs one pass of online
// softmax on the tensor cores (mma.sync m16n8k16: A = the g query rows padded
// to 16, B = K rows via ldmatrix; then A = P, B = V rows via ldmatrix.trans).
// Every logit goes to an L2-resident scratch; when a group leaves a row it
// combines its four warps, writes one (max, sum, O) partial and appends its
// index to the row's partial list. No CTA waits on another.
// decode_finish_kernel (CTAs per row slice): combines the row's listed
// partials into the attention output, applies the exact probabilities to A,
// picks the eviction and updates the row's meta data.
constexpr int kTcSlots = 64;  // slots per TMA tile
constexpr int kCH = 128;      // slots per work item
constexpr int kSkStages = 6;
constexpr int kGroups = 3;  // consumer groups of four warps; group k takes the tiles with it % 3 == k
constexpr int kSkConsumers = 4 * kGroups;
constexpr int kSkThreads = (kSkConsumers + 1) * 32;
constexpr int kTcMaxG = 8;                     // query heads per KV head on the tensor-core path
constexpr int kQBytes = kTcMaxG * 128 * 2;     // staged query rows per stage
constexpr int kFinThreads = 1024;
constexpr int kFinSlots = 2048;  // slots per finishing CTA

__device__ __forceinline__ uint32_t swz(uint32_t tile, int slot, int dcol) {
  const int box = dcol >> 6, chunk = (dcol & 63) >> 3;
  return tile + box * (kTcSlots * 128) + slot * 128 + ((chunk ^ (slot & 7)) << 4);
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }


__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Decode scratch inside kv_cache.scratch.
struct DecScratch {
  int* n_items;   // [1]
  int* item_off;  // [rows + 1] first item of each row
  int2* items;    // [max_items] (row, chunk)
  float* part;    // [max_items * groups][stride]: (max[G], sum[G], O[G][d]) per (segment-first item, group)
  float* logits;  // [total_slots][G] logits in log2 units
  int* tickets;   // [rows] finished slices of the current step, reset by the row's last slice
  int* plist_n;   // [rows] partials written for the row in the current step (reset by its last slice)
  int* plist;     // [rows][max_per_row * groups] their slot indices
  int4* bests;    // [rows][max_slices] eviction candidate per slice: (A bits, pos, slot, -)
  int max_items, max_per_row, stride, max_slices;
};

size_t dec_scratch_layout(int rows, int G, int d, int capb, long long total_slots, char* base, DecScratch* sc) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int per_row = (capb + kCH - 1) / kCH;
  const int max_items = rows * per_row;
  const int stride = (2 * G + G * d + 3) & ~3;
  size_t off = 0;
  const size_t o_n = off;
  off += 256;
  const size_t o_ioff = off;
  off += al((size_t)(rows + 1) * 4);
  const size_t o_items = off;
  off += al((size_t)max_items * 8);
  const size_t o_part = off;
  off += al((size_t)max_items * kGroups * stride * 4);
  const size_t o_log = off;
  off += al((size_t)total_slots * G * 4);
  const int max_slices = (capb + kFinSlots - 1) / kFinSlots;
  const size_t o_tk = off;
  off += al((size_t)rows * 4);
  const size_t o_pn = off;
  off += al((size_t)rows * 4);
  const size_t o_pl = off;
  off += al((size_t)rows * per_row * kGroups * 4);
  const size_t o_best = off;
  off += al((size_t)rows * max_slices * 16);
  if (sc && base) {
    sc->n_items = reinterpret_cast<int*>(base + o_n);
    sc->item_off = reinterpret_cast<int*>(base + o_ioff);
    sc->items = reinterpret_cast<int2*>(base + o_items);
    sc->part = reinterpret_cast<float*>(base + o_part);
    sc->logits = reinterpret_cast<float*>(base + o_log);
    sc->tickets = reinterpret_cast<int*>(base + o_tk);
    sc->plist_n = reinterpret_cast<int*>(base + o_pn);
    sc->plist = reinterpret_cast<int*>(base + o_pl);
    sc->bests = reinterpret_cast<int4*>(base + o_best);
    sc->max_slices = max_slices;
    sc->max_items = max_items;
    sc->max_per_row = per_row;
    sc->stride = stride;
  }
  return off;
}

struct SkArgs {
  DecArgs a;
  DecScratch sc;
  int nk;  // 64-element boxes per row (d / 64)
  unsigned long long limit_ns;
};

// What the producer learns about a tile and hands to the consumers.
struct TileHdr {
  int row, u, st0, c1, count, next, steps, cap;  // row = -1: no more tiles for this group
  long long base;
};

template <int D>
__global__ void __launch_bounds__(kSkThreads, 1) decode_attn_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const SkArgs P) {
  constexpr int NDC = D / 16;                       // 16-wide chunks of d
  constexpr int TILE = kTcSlots * D * 2;            // bytes of one K or V tile
  constexpr int STAGE = 2 * TILE + kQBytes;         // K tile, V tile, query rows
  const DecArgs& a = P.a;
  const DecScratch& sc = P.sc;
  const int G = a.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q_bytes = G * D * 2;

  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  float* o_s = reinterpret_cast<float*>(ring + kSkStages * STAGE);  // [groups][G][D]
  __shared__ uint64_t full[kSkStages], empty[kSkStages];
  __shared__ TileHdr hdr[kSkStages];
  __shared__ float red_m[kSkConsumers][kTcMaxG], red_l[kSkConsumers][kTcMaxG];
  __shared__ int abort_s;

  if (tid == 0) {
    for (int i = 0; i < kSkStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    abort_s = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  for (int i = tid; i < kGroups * G * D; i += kSkThreads) o_s[i] = 0.f;
  pdl_wait();  // the previous step's finish has written meta and read the scratch
  pdl_launch_dependents();
  __syncthreads();
  const Guard gd{&abort_s, a.status, P.limit_ns};
  const int n_items = *sc.n_items;
  const int u0 = (int)((long long)n_items * blockIdx.x / gridDim.x);
  const int u1 = (int)((long long)n_items * (blockIdx.x + 1) / gridDim.x);

  if (warp == kSkConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t stream_policy = make_policy_evict_first();  // K/V are read once per step
      bool issued[kSkStages] = {};
      uint32_t par[kSkStages] = {};
      bool aborted = false;
      int it = 0;
      int2 item = u0 < u1 ? sc.items[u0] : make_int2(0, 0);
      int cur = -1, cap = 0, count = 0, next = 0, steps = 0;
      long long base = 0;
      for (int u = u0; u < u1 && !aborted; ++u) {
        const int row = item.x, chunk = item.y;
        if (u + 1 < u1) item = sc.items[u + 1];  // in flight while this item is issued
        if (row != cur) {  // a row's state is fixed for the whole step: load it once
          cur = row;
          base = a.slot_off[row];
          cap = (int)(a.slot_off[row + 1] - base);
          const int* mrow = a.meta + (long long)row * 8;
          count = mrow[0];
          next = mrow[1];
          steps = mrow[2];
        }
        const int c0 = chunk * kCH, c1 = min(c0 + kCH, cap);
        const int nt = (c1 - c0 + kTcSlots - 1) / kTcSlots;
        const void* qsrc = static_cast<const __nv_bfloat16*>(a.q) + (long long)row * G * D;
        for (int t = 0; t < nt; ++t, ++it) {
          const int st = it % kSkStages;
          if (it >= kSkStages && !wait_bounded(&empty[st], ((it / kSkStages) - 1) & 1, gd)) {
            aborted = true;
            break;
          }
          TileHdr h;
          h.row = row;
          h.u = u;
          h.st0 = c0 + t * kTcSlots;
          h.c1 = c1;
          h.count = count;
          h.next = next;
          h.steps = steps;
          h.cap = cap;
          h.base = base;
          hdr[st] = h;
          uint8_t* stage = ring + st * STAGE;
          mbar_arrive_expect_tx(&full[st], 2 * TILE + q_bytes);
          const int y = (int)(base + h.st0);
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_2d_hint(stage + bx * kTcSlots * 128, &tmK, &full[st], bx * 64, y, stream_policy);
            tma_load_2d_hint(stage + TILE + bx * kTcSlots * 128, &tmV, &full[st], bx * 64, y, stream_policy);
          }
          bulk_load(stage + 2 * TILE, qsrc, q_bytes, &full[st]);
          issued[st] = true;
          par[st] = (it / kSkStages) & 1;
        }
      }
      // one sentinel stage per consumer group: a header with row = -1, no data
      for (int k = 0; k < kGroups && !aborted; ++k, ++it) {
        const int st = it % kSkStages;
        if (it >= kSkStages && !wait_bounded(&empty[st], ((it / kSkStages) - 1) & 1, gd)) {
          aborted = true;
          break;
        }
        hdr[st].row = -1;
        mbar_arrive(&full[st]);
      }
      if (aborted || abort_s)
        for (int st = 0; st < kSkStages; ++st)
          if (issued[st]) wait_drain(&full[st], par[st], P.limit_ns);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g0 = lane >> 2, q4 = lane & 3;  // this lane's query row and column pair
  const bool g_ok = g0 < G;
  const int m_ = lane >> 3, r_ = lane & 7;
  const int grp = warp >> 2;          // tiles with it % kGroups == grp
  const int wslot = (warp & 3) * 16;  // this warp's 16 slots of a tile
  const uint64_t keep_policy = make_policy_evict_last();  // logits are read back by the finish kernel
  float* og = o_s + grp * G * D;
  bool aborted = false;
  int cur_row = -1, seg_u = -1;
  uint32_t qa[NDC][2];  // A fragments of the query rows (rows 8..15 of the m16 tile are zero)
  float m0 = -INFINITY, l0 = 0.f;
  float o[2 * NDC][2];  // O[g0][8 i + 2 q4 + {0,1}]
#pragma unroll
  for (int i = 0; i < 2 * NDC; ++i) o[i][0] = o[i][1] = 0.f;

  // walk the stages in issue order; this group takes the tiles with it % kGroups == grp
  for (int it = grp;; it += kGroups) {
    const int st = it % kSkStages;
    const bool got = !aborted && wait_bounded(&full[st], (it / kSkStages) & 1, gd);
    if (!got) aborted = true;
    const int hrow = got ? hdr[st].row : -1;  // -1: sentinel (or abort), the CTA's tiles are done
    if (hrow != cur_row || hrow < 0) {
      if (cur_row >= 0) {
        // leaving a row: this group's running (max, sum, O) becomes one partial at
        // (first item of the segment, group), listed for the row's finish
        float ls0 = l0;
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) ls0 += __shfl_xor_sync(0xffffffffu, ls0, off);
        if (q4 == 0 && g_ok) {
          red_m[warp][g0] = m0;
          red_l[warp][g0] = ls0;
        }
        named_bar_sync(1 + grp, 128);
        float M0 = -INFINITY;
        if (g_ok)
          for (int w = 0; w < 4; ++w) M0 = fmaxf(M0, red_m[grp * 4 + w][g0]);
        const float f0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M0);
        if (g_ok) {
#pragma unroll
          for (int i = 0; i < 2 * NDC; ++i) {
            const int col = i * 8 + q4 * 2;
            atomicAdd(&og[g0 * D + col], o[i][0] * f0);
            atomicAdd(&og[g0 * D + col + 1], o[i][1] * f0);
          }
        }
        named_bar_sync(1 + grp, 128);
        float* part = sc.part + ((long long)seg_u * kGroups + grp) * sc.stride;
        const int gt = tid - grp * 128;  // thread index within the group
        if (gt < G) {
          float M = -INFINITY;
          for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[grp * 4 + w][gt]);
          float Ls = 0.f;
          for (int w = 0; w < 4; ++w)
            if (red_m[grp * 4 + w][gt] > -INFINITY)
              Ls += red_l[grp * 4 + w][gt] * ex2_approx(red_m[grp * 4 + w][gt] - M);
          part[gt] = M;
          part[G + gt] = Ls;
        }
        for (int i = gt; i < G * D; i += 128) {
          part[2 * G + i] = og[i];
          og[i] = 0.f;
        }
        if (gt == 0) {
          const int k = atomicAdd(&sc.plist_n[cur_row], 1);
          if (k < sc.max_per_row * kGroups) sc.plist[(long long)cur_row * sc.max_per_row * kGroups + k] = seg_u * kGroups + grp;
        }
        named_bar_sync(1 + grp, 128);
        m0 = -INFINITY;
        l0 = 0.f;
#pragma unroll
        for (int i = 0; i < 2 * NDC; ++i) o[i][0] = o[i][1] = 0.f;
      }
      if (hrow < 0) break;
      cur_row = hrow;
      seg_u = hdr[st].u;
      // query fragments from the staged [G][D] rows (rows >= G are zero)
      const uint32_t qs = smem_u32(ring + st * STAGE) + 2 * TILE;
      const int qrow = lane & 7;
#pragma unroll
      for (int dc = 0; dc < NDC; ++dc) {
        uint32_t r0, r1, r2, r3;
        const uint32_t addr = qs + (uint32_t)((qrow < G ? qrow : 0) * D + dc * 16 + (lane >> 4) * 8) * 2;
        ldsm_x4(addr, r0, r1, r2, r3);
        qa[dc][0] = g_ok ? r0 : 0u;
        qa[dc][1] = g_ok ? r2 : 0u;
      }
    }
    const TileHdr h = hdr[st];
    uint8_t* stage = ring + st * STAGE;
    const uint32_t ktile = smem_u32(stage), vtile = ktile + TILE;
    const int n = h.count + 1;
    const bool row_ok = h.count >= 0 && h.count < h.cap && h.next >= 0 && h.next < h.cap;
    const int next = h.next;
    const long long base = h.base;
    if (row_ok && next >= h.st0 + wslot && next < h.st0 + wslot + 16 && next < h.c1) {
      // the appended token: patch its K and V rows into the tile, write them to the cache
      const int r = next - h.st0;
      const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(a.k) + (long long)h.row * D;
      const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(a.v) + (long long)h.row * D;
      if (lane < D / 8) {
        const uint4 kv = *reinterpret_cast<const uint4*>(kin + lane * 8);
        const uint4 vv = *reinterpret_cast<const uint4*>(vin + lane * 8);
        *reinterpret_cast<uint4*>(stage + (swz(ktile, r, lane * 8) - ktile)) = kv;
        *reinterpret_cast<uint4*>(stage + (swz(vtile, r, lane * 8) - ktile)) = vv;
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Kc) + (base + next) * D)[lane] = kv;
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Vc) + (base + next) * D)[lane] = vv;
      }
      if (lane == 0) a.pos[base + next] = row_len(a.map, h.row) + h.steps;
      fence_proxy_async();
      __syncwarp();
    }
    // logits S = Q K^T for this warp's 16 slots (even and odd d-chunks accumulate
    // separately: four independent MMA chains)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int dc = 0; dc < NDC; ++dc) {
      uint32_t b00, b01, b10, b11;
      ldsm_x4(swz(ktile, wslot + (m_ >> 1) * 8 + r_, dc * 16 + (m_ & 1) * 8), b00, b01, b10, b11);
      const uint32_t af[4] = {qa[dc][0], 0u, qa[dc][1], 0u};
      if (dc & 1) {
        mma16816(t0, af, b00, b01);
        mma16816(t1, af, b10, b11);
      } else {
        mma16816(s0, af, b00, b01);
        mma16816(s1, af, b10, b11);
      }
    }
    const int jb = h.st0 + wslot + q4 * 2;  // slots jb, jb+1 (n-tile 0) and jb+8, jb+9 (n-tile 1)
    float x[4];                              // row g0 at those four slots
    x[0] = s0[0] + t0[0];
    x[1] = s0[1] + t0[1];
    x[2] = s1[0] + t1[0];
    x[3] = s1[1] + t1[1];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = jb + (e & 1) + (e >> 1) * 8;
      const bool valid = row_ok && j < n && j < h.c1;
      x[e] = valid ? x[e] * a.scale2 : -INFINITY;
      if (valid && g_ok) st_f32_hint(sc.logits + (base + j) * G + g0, x[e], keep_policy);
    }
    // online softmax update of this warp's running (max, sum, O)
    float tm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
    const float nm = fmaxf(m0, tm);
    const float vm = nm == -INFINITY ? 0.f : nm;
    if (__any_sync(0xffffffffu, nm != m0)) {  // rescale only when a running max moved
      const float sc0 = ex2_approx(m0 - vm);
      l0 *= sc0;
#pragma unroll
      for (int i = 0; i < 2 * NDC; ++i) {
        o[i][0] *= sc0;
        o[i][1] *= sc0;
      }
    }
    m0 = nm;
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = ex2_approx(x[e] - vm);
      l0 += p[e];
    }
    const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
#pragma unroll
    for (int dn = 0; dn < NDC; ++dn) {
      uint32_t b0a, b1a, b0b, b1b;
      ldsm_x4_t(swz(vtile, wslot + (m_ & 1) * 8 + r_, dn * 16 + (m_ >> 1) * 8), b0a, b1a, b0b, b1b);
      float c0[4] = {o[2 * dn][0], o[2 * dn][1], 0.f, 0.f};
      float c1[4] = {o[2 * dn + 1][0], o[2 * dn + 1][1], 0.f, 0.f};
      mma16816(c0, pa, b0a, b1a);
      mma16816(c1, pa, b0b, b1b);
      o[2 * dn][0] = c0[0];
      o[2 * dn][1] = c0[1];
      o[2 * dn + 1][0] = c1[0];
      o[2 * dn + 1][1] = c1[1];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (aborted) abort_s = 1;
}

// Finish of one decode step, one CTA per (row, slice of kFinSlots slots):
// the row's log-denominators from the partials the attention kernel listed
// for the row, this slice's share of the attention output, the exact
// probabilities p = exp2(logit - lse) added into the decayed scores A of the
// slice's slots, and the slice's best eviction candidate. The row's last
// slice to finish (atomic ticket, no waiting) picks the eviction, updates
// the row's meta data and clears the row's partial list.
__global__ void __launch_bounds__(kFinThreads) decode_finish_kernel(const SkArgs P) {
  const DecArgs& a = P.a;
  const DecScratch& sc = P.sc;
  const int G = a.G, d = a.d, E = G * d;
  const int row = blockIdx.x / sc.max_slices, slice = blockIdx.x % sc.max_slices;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kMaxParts = 32;  // partials combined per row (more are folded serially below)
  __shared__ int plist_s[kMaxParts];
  __shared__ float pm_s[kMaxParts][kTcMaxG], pl_s[kMaxParts][kTcMaxG];
  __shared__ float Ms[kTcMaxG], Li[kTcMaxG], lse_s[kTcMaxG];
  __shared__ Best bw[kFinThreads / 32];
  __shared__ int last_s;

  pdl_wait();  // the attention kernel's partials and logits are complete
  pdl_launch_dependents();
  // round 1: the row's state and its list of partials
  int32_t* meta = a.meta + (long long)row * 8;
  const int count = meta[0], next = meta[1], steps = meta[2], count0 = meta[4];
  const int nr_all = sc.plist_n[row];
  const int n = count + 1;
  const int nsl = (n + kFinSlots - 1) / kFinSlots;
  if (slice >= nsl) return;  // uniform over the CTA
  const long long base = a.slot_off[row];
  const int cap = (int)(a.slot_off[row + 1] - base);
  const int bb = a.b[row];
  const int pos_new = row_len(a.map, row) + steps;
  const int Mr = (a.recent_pct * bb) / 100;
  const int appended = steps + 1;
  const bool evict = n > bb;
  const bool ok = count < cap && next >= 0 && next < cap && (!evict || bb >= a.T + Mr);
  const int nr = min(nr_all, sc.max_per_row * kGroups);
  const int* plist = sc.plist + (long long)row * sc.max_per_row * kGroups;
  if (tid < min(nr, kMaxParts)) plist_s[tid] = plist[tid];
  // round 2: this thread's slots (A, pos, logits) and the eviction threshold
  constexpr int U = kFinSlots / kFinThreads;
  float Av[U], lgv[U][kTcMaxG];
  int pv[U];
#pragma unroll
  for (int k = 0; k < U; ++k) {
    const int j = slice * kFinSlots + k * kFinThreads + tid;
    Av[k] = 0.f;
    pv[k] = 0;
#pragma unroll
    for (int g = 0; g < kTcMaxG; ++g) lgv[k][g] = -INFINITY;
    if (ok && j < n) {
      Av[k] = a.A[base + j];
      pv[k] = a.pos[base + j];
      const float* lg = sc.logits + (base + j) * G;
      if (G == 8) {
        const float4 v0 = *reinterpret_cast<const float4*>(lg);
        const float4 v1 = *reinterpret_cast<const float4*>(lg + 4);
        lgv[k][0] = v0.x; lgv[k][1] = v0.y; lgv[k][2] = v0.z; lgv[k][3] = v0.w;
        lgv[k][4] = v1.x; lgv[k][5] = v1.y; lgv[k][6] = v1.z; lgv[k][7] = v1.w;
      } else {
#pragma unroll
        for (int g = 0; g < kTcMaxG; ++g)
          if (g < G) lgv[k][g] = lg[g];
      }
    }
  }
  const int pos_thr = (!ok || appended >= Mr) ? pos_new - Mr + 1 : a.pos[base + max(0, count0 - (Mr - appended))];
  __syncthreads();
  // the partials' (max, sum) per query head
  const int nr_s = min(nr, kMaxParts);
  if (tid < nr_s * G) {
    const int k = tid / G, g = tid % G;
    const float* pc = sc.part + (long long)plist_s[k] * sc.stride;
    pm_s[k][g] = pc[g];
    pl_s[k][g] = pc[G + g];
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int k = 0; k < nr_s; ++k) M = fmaxf(M, pm_s[k][tid]);
    for (int k = kMaxParts; k < nr; ++k) M = fmaxf(M, sc.part[(long long)plist[k] * sc.stride + tid]);
    float Ls = 0.f;
    for (int k = 0; k < nr_s; ++k)
      if (pm_s[k][tid] > -INFINITY) Ls += pl_s[k][tid] * exp2f(pm_s[k][tid] - M);
    for (int k = kMaxParts; k < nr; ++k) {
      const float* pc = sc.part + (long long)plist[k] * sc.stride;
      if (pc[tid] > -INFINITY) Ls += pc[G + tid] * exp2f(pc[tid] - M);
    }
    Ms[tid] = M;
    Li[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
    lse_s[tid] = M + log2f(Ls);
  }
  __syncthreads();
  // round 3: this slice's share of the attention output
  {
    const int e0 = (int)((long long)E * slice / nsl), e1 = (int)((long long)E * (slice + 1) / nsl);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (long long)row * E;
    for (int i = e0 + tid; i < e1; i += kFinThreads) {
      const int g = i / d;
      float acc = 0.f;
#pragma unroll 4
      for (int k = 0; k < nr; ++k) {
        const int slot = k < kMaxParts ? plist_s[k] : plist[k];
        const float mc = k < kMaxParts ? pm_s[k][g] : sc.part[(long long)slot * sc.stride + g];
        const float w = mc > -INFINITY ? exp2f(mc - Ms[g]) : 0.f;
        acc += w * sc.part[(long long)slot * sc.stride + 2 * G + i];
      }
      out[i] = __float2bfloat16_rn(acc * Li[g]);
    }
  }
  // the exact probabilities into A (data already in registers), this slice's candidate
  const bool timed_out = (*reinterpret_cast<volatile int32_t*>(a.status) & KV_DEV_TIMEOUT) != 0;
  Best best{INFINITY, -1, -1};
  if (ok && !timed_out) {
    float lse[kTcMaxG];
#pragma unroll
    for (int g = 0; g < kTcMaxG; ++g) lse[g] = g < G ? lse_s[g] : 0.f;
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int j = slice * kFinSlots + k * kFinThreads + tid;
      if (j < n) {
        float psum = 0.f;
#pragma unroll
        for (int g = 0; g < kTcMaxG; ++g)
          if (g < G) psum += ex2_approx(lgv[k][g] - lse[g]);
        const float Anew = (j == next ? 0.f : a.gamma * Av[k]) + psum;
        a.A[base + j] = Anew;
        const int pj = j == next ? pos_new : pv[k];
        if (j >= a.T && pj < pos_thr) {
          const Best c{Anew, pj, j};
          if (better(c, best)) best = c;
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Best y;
    y.A = __shfl_xor_sync(0xffffffffu, best.A, off);
    y.pos = __shfl_xor_sync(0xffffffffu, best.pos, off);
    y.slot = __shfl_xor_sync(0xffffffffu, best.slot, off);
    if (better(y, best)) best = y;
  }
  if (lane == 0) bw[warp] = best;
  __syncthreads();
  if (warp == 0) {
    Best bst = lane < kFinThreads / 32 ? bw[lane] : Best{INFINITY, -1, -1};
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      Best y;
      y.A = __shfl_xor_sync(0xffffffffu, bst.A, off);
      y.pos = __shfl_xor_sync(0xffffffffu, bst.pos, off);
      y.slot = __shfl_xor_sync(0xffffffffu, bst.slot, off);
      if (better(y, bst)) bst = y;
    }
    if (lane == 0) {
      sc.bests[(long long)row * sc.max_slices + slice] = make_int4(__float_as_int(bst.A), bst.pos, bst.slot, 0);
      __threadfence();
      last_s = atomicAdd(&sc.tickets[row], 1) == nsl - 1;
    }
  }
  __syncthreads();
  if (!last_s || tid != 0) return;
  // the row's last slice: reduce the candidates, evict, update meta, clear the list
  __threadfence();
  Best bst{INFINITY, -1, -1};
  for (int k = 0; k < nsl; ++k) {
    const volatile int* v = reinterpret_cast<volatile int*>(sc.bests + (long long)row * sc.max_slices + k);
    const Best c{__int_as_float(v[0]), v[1], v[2]};
    if (better(c, bst)) bst = c;
  }
  if (!ok || nr_all > sc.max_per_row * kGroups) {
    atomicOr(a.status, !ok ? KV_DEV_BUDGET : KV_DEV_CAPACITY);
  } else if (!timed_out) {
    if (evict && bst.slot >= 0) {
      meta[0] = bb;
      meta[1] = bst.slot;
      meta[3] = bst.slot;
    } else {
      meta[0] = n;
      meta[1] = n;
      meta[3] = -1;
    }
    meta[2] = steps + 1;
  }
  sc.tickets[row] = 0;
  sc.plist_n[row] = 0;
}

// Builds the work items of every row (rows cut into kCH-slot chunks) and
// clears the row tickets and partial lists; one block.
__global__ void decode_items_kernel(int n_rows, const int64_t* __restrict__ slot_off, DecScratch sc,
                                    int32_t* __restrict__ status) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_rows; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int own = 0;
    if (i < n_rows) {
      const long long cap = slot_off[i + 1] - slot_off[i];
      own = (int)((cap + kCH - 1) / kCH);
      if (own > sc.max_per_row) {
        atomicOr(status, KV_DEV_CAPACITY);
        own = sc.max_per_row;
      }
    }
    int v = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    int wb = 0;
    for (int k = 0; k < warp; ++k) wb += warp_tot[k];
    const int incl = carry + wb + v;
    if (i < n_rows) {
      sc.tickets[i] = 0;
      sc.plist_n[i] = 0;
      sc.item_off[i] = incl - own;
      for (int c = 0; c < own; ++c) sc.items[incl - own + c] = make_int2(i, c);
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    sc.item_off[n_rows] = carry;
    *sc.n_items = carry;
  }
}

// One block per row: A = 0 on the row's slots, meta reset, budget check.
__global__ void decode_init_kernel(const int64_t* __restrict__ slot_off, const int32_t* __restrict__ b, int T,
                                   int recent_pct, float* __restrict__ A, int32_t* __restrict__ meta,
                                   int32_t* __restrict__ status) {
  const int row = blockIdx.x;
  const long long s0 = slot_off[row], s1 = slot_off[row + 1];
  for (long long i = s0 + threadIdx.x; i < s1; i += blockDim.x) A[i] = 0.f;
  if (threadIdx.x == 0) {
    const int bb = b[row];
    int32_t* m = meta + (long long)row * 8;
    m[0] = bb;
    m[1] = bb;
    m[2] = 0;
    m[3] = -1;
    m[4] = bb;
    m[5] = m[6] = m[7] = 0;
    if (bb < T + (recent_pct * bb) / 100 || s1 - s0 != (long long)bb + 1) atomicOr(status, KV_DEV_BUDGET);
  }
}

// Largest b_i + 1 a row can have: b_h <= min(L, B - (H - 1) w) since every
// other head of the layer keeps at least w.
int cap_bound(const kv_shape& sh, const RowMap& m, const kv_params& p) {
  long long mx = 0;
  for (int s = 0; s < m.n_seq; ++s) {
    const long long L = m.L[s];
    const long long B = ((long long)p.budget_pct * L * sh.n_kv_heads) / 100;
    const long long bmax = std::min(L, B - (long long)(sh.n_kv_heads - 1) * sh.w);
    mx = std::max(mx, bmax + 1);
  }
  return (int)mx;
}

}  // namespace

int cap_bound_of(const kv_shape& sh, const RowMap& m, const kv_params& p) { return cap_bound(sh, m, p); }

size_t decode_scratch_bytes(const kv_shape& sh, const RowMap& m, const kv_params& p, long long total_slots) {
  return dec_scratch_layout(m.n_rows, sh.group, sh.head_dim, cap_bound(sh, m, p), total_slots, nullptr, nullptr);
}

static long long cache_slots(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c) {
  return c.total_slots > 0 ? c.total_slots : kv_total_slots(&sh, m.L, m.n_seq, &p);
}

int launch_decode_init(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c,
                       cudaStream_t st) {
  decode_init_kernel<<<m.n_rows, 256, 0, st>>>(c.slot_off, c.b, p.sinks_T, p.recent_pct, c.A, c.meta, c.status);
  if (sh.dtype == KV_BF16 && sh.group <= kTcMaxG) {
    const long long total = cache_slots(sh, m, p, c);
    DecScratch sc;
    const size_t need =
        dec_scratch_layout(m.n_rows, sh.group, sh.head_dim, cap_bound(sh, m, p), total, (char*)c.scratch, &sc);
    if (!c.scratch || c.scratch_bytes < need) return KV_ERR_WORKSPACE;
    decode_items_kernel<<<1, 1024, 0, st>>>(m.n_rows, c.slot_off, sc, c.status);
  }
  return cuda_status(cudaGetLastError());
}

int launch_decode(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c, const void* q_t,
                  const void* k_t, const void* v_t, void* out, cudaStream_t st) {
  if (sh.group > kMaxG) return KV_ERR_ARG;
  const int capb = cap_bound(sh, m, p);
  DecArgs a;
  a.map = m;
  a.G = sh.group;
  a.d = sh.head_dim;
  a.scale2 = (float)(1.4426950408889634 / std::sqrt((double)sh.head_dim));
  a.gamma = p.gamma;
  a.T = p.sinks_T;
  a.recent_pct = p.recent_pct;
  a.q = q_t;
  a.k = k_t;
  a.v = v_t;
  a.out = out;
  a.Kc = c.Kc;
  a.Vc = c.Vc;
  a.A = c.A;
  a.pos = c.pos;
  a.slot_off = c.slot_off;
  a.b = c.b;
  a.meta = c.meta;
  a.status = c.status;
  cudaError_t e;
  if (sh.dtype == KV_BF16 && sh.group <= kTcMaxG) {
    const long long total = cache_slots(sh, m, p, c);
    SkArgs P;
    P.a = a;
    P.a.C = 1;
    P.a.S_cap = 0;
    const size_t need = dec_scratch_layout(m.n_rows, sh.group, sh.head_dim, capb, total, (char*)c.scratch, &P.sc);
    if (!c.scratch || c.scratch_bytes < need) return KV_ERR_WORKSPACE;
    P.nk = sh.head_dim / 64;
    P.limit_ns = kWaitLimitNs;
    const int stage_bytes = 2 * kTcSlots * sh.head_dim * 2 + kQBytes;
    const size_t smem = 1024 + (size_t)kSkStages * stage_bytes + (size_t)kGroups * sh.group * sh.head_dim * 4;
    CUtensorMap tmK, tmV;
    if (!encode_rows_bf16(&tmK, c.Kc, sh.head_dim, total, kTcSlots)) return KV_ERR_CUDA;
    if (!encode_rows_bf16(&tmV, c.Vc, sh.head_dim, total, kTcSlots)) return KV_ERR_CUDA;
    const size_t fsmem = 0;
    auto attn = sh.head_dim == 128 ? decode_attn_kernel<128> : decode_attn_kernel<64>;
    if (cudaFuncSetAttribute(attn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return KV_ERR_ARG;
    // both launches may start while the kernel before them drains (programmatic
    // dependent launch); each waits (griddepcontrol.wait) before touching memory
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(sm_count());
    c1.blockDim = dim3(kSkThreads);
    c1.dynamicSmemBytes = smem;
    c1.stream = st;
    c1.attrs = pdl;
    c1.numAttrs = 1;
    e = cudaLaunchKernelEx(&c1, attn, tmK, tmV, P);
    if (e != cudaSuccess) return KV_ERR_CUDA;
    cudaLaunchConfig_t c2 = c1;
    c2.gridDim = dim3(m.n_rows * P.sc.max_slices);
    c2.blockDim = dim3(kFinThreads);
    c2.dynamicSmemBytes = fsmem;
    e = cudaLaunchKernelEx(&c2, decode_finish_kernel, P);
  } else {
    int C = 8;
    while (C > 1 && (capb + C - 1) / C < 128) C >>= 1;
    a.C = C;
    a.S_cap = (capb + C - 1) / C;
    const size_t smem = ((size_t)sh.group * a.S_cap + 2 * (size_t)sh.group * sh.head_dim) * sizeof(float);
    if (smem > 200 * 1024) return KV_ERR_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(m.n_rows * C);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (sh.dtype == KV_BF16) {
      cudaFuncSetAttribute(decode_simple_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           200 * 1024);
      e = cudaLaunchKernelEx(&cfg, decode_simple_kernel<__nv_bfloat16>, a);
    } else {
      cudaFuncSetAttribute(decode_simple_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      e = cudaLaunchKernelEx(&cfg, decode_simple_kernel<float>, a);
    }
  }
  return cuda_status(e);
}

}  // namespace kvc
