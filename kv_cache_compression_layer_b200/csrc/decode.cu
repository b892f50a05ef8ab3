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
// bf16 caches: tensor-core decode.
//
// Per row a cluster of C CTAs; CTA c owns slots [c S, c S + S). Warp 4
// streams the CTA's slots as 64-slot tiles (K tiles first, then V tiles)
// through a 4-stage ring with TMA (128-byte swizzled boxes, so the
// ldmatrix reads below are bank-conflict free). Warps 0-3 each own 16 slots
// of a tile:
//   phase 1  S = Q K^T with mma.sync m16n8k16 (A = the g query rows, padded
//            to 16; B = K rows via ldmatrix), logits (log2 units) kept in
//            shared memory, running max per query head;
//   phase 2  CTA max per query head;
//   phase 3  P = exp2(S - max) rebuilt as mma A fragments from shared
//            memory, O += P V (B = V rows via ldmatrix.trans), row sums;
// then the CTAs combine (max, sum, O) through distributed shared memory,
// each writing a slice of the output, apply the exact probabilities to A and
// reduce the eviction candidate. The appended token's row is patched into the
// tile (and written to the cache) by the warp that owns its slot.
constexpr int kTcSlots = 64;
constexpr int kTcStages = 4;
constexpr int kTcConsumers = 4;
constexpr int kTcThreads = (kTcConsumers + 1) * 32;

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

struct TcDec {
  DecArgs a;
  int S_pad;  // row stride of the logit buffer
  int nk;     // 64-element boxes per row (d / 64)
  unsigned long long limit_ns;
};

__global__ void __launch_bounds__(kTcThreads) decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ CUtensorMap tmV,
                                                                const TcDec P) {
  const DecArgs& a = P.a;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / a.C;
  const int G = a.G, d = a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile_bytes = kTcSlots * d * 2;

  extern __shared__ uint8_t dsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* xs = reinterpret_cast<float*>(smem + kTcStages * tile_bytes);  // [G][S_pad] logits (log2 units)
  float* o_s = xs + G * P.S_pad;                                        // [G][d]
  __shared__ uint64_t full[kTcStages], empty[kTcStages];
  __shared__ float m_s[kMaxG], l_s[kMaxG], lse_s[kMaxG], M_s[kMaxG], Li_s[kMaxG];
  __shared__ float red_m[kTcConsumers][kMaxG];
  __shared__ float mr_s[8][kMaxG];
  __shared__ Best bw[kTcConsumers + 1];
  __shared__ Best best_s;
  __shared__ int abort_s;

  const int L = row_len(a.map, row);
  const long long base = a.slot_off[row];
  const int cap = (int)(a.slot_off[row + 1] - base);
  const int bb = a.b[row];
  int32_t* meta = a.meta + (long long)row * 8;
  const int count = meta[0], next = meta[1], steps = meta[2], count0 = meta[4];
  const int n = count + 1;
  const int pos_new = L + steps;
  const int M = (a.recent_pct * bb) / 100;
  const int appended = steps + 1;
  const bool evict = n > bb;
  const int S = (cap + a.C - 1) / a.C;
  const int j0 = rank * S, j1 = min(j0 + S, n);
  const bool ok = S <= a.S_cap && count < cap && (!evict || bb >= a.T + M);
  const int cnt = ok ? max(0, j1 - j0) : 0;
  const int nt = (cnt + kTcSlots - 1) / kTcSlots;
  if (!ok && rank == 0 && tid == 0) atomicOr(a.status, S > a.S_cap ? KV_DEV_CAPACITY : KV_DEV_BUDGET);

  const __nv_bfloat16* qin = static_cast<const __nv_bfloat16*>(a.q) + (long long)row * G * d;
  const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(a.k) + (long long)row * d;
  const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(a.v) + (long long)row * d;
  __nv_bfloat16* Kc = static_cast<__nv_bfloat16*>(a.Kc) + base * d;
  __nv_bfloat16* Vc = static_cast<__nv_bfloat16*>(a.Vc) + base * d;
  float* A = a.A + base;
  int32_t* pos = a.pos + base;

  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kTcConsumers);
    }
    abort_s = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < G * d; i += kTcThreads) o_s[i] = 0.f;
  if (tid < kMaxG) l_s[tid] = 0.f;
  __syncthreads();
  const Guard gd{&abort_s, a.status, P.limit_ns};
  const int owner_tile = (next >= j0 && next < j0 + cnt) ? (next - j0) / kTcSlots : -1;

  if (warp == kTcConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      bool issued[kTcStages] = {false, false, false, false};
      uint32_t par[kTcStages] = {0, 0, 0, 0};
      bool aborted = false;
      for (int it = 0; it < 2 * nt; ++it) {
        const int st = it % kTcStages;
        if (it >= kTcStages && !wait_bounded(&empty[st], ((it / kTcStages) - 1) & 1, gd)) {
          aborted = true;
          break;
        }
        mbar_arrive_expect_tx(&full[st], tile_bytes);
        const int t = it < nt ? it : it - nt;
        const int y = (int)(base + j0 + t * kTcSlots);
        for (int bx = 0; bx < P.nk; ++bx)
          tma_load_2d(ring + st * tile_bytes + bx * kTcSlots * 128, it < nt ? &tmK : &tmV, &full[st], bx * 64, y);
        issued[st] = true;
        par[st] = (it / kTcStages) & 1;
      }
      if (aborted || abort_s)
        for (int st = 0; st < kTcStages; ++st)
          if (issued[st]) wait_drain(&full[st], par[st], P.limit_ns);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int g0 = lane >> 2, q4 = lane & 3;
    const int ndc = d / 16;
    uint32_t qa[8][4];
#pragma unroll
    for (int dc = 0; dc < 8; ++dc) {
      if (dc < ndc) {
        const int c = dc * 16 + q4 * 2;
        qa[dc][0] = g0 < G ? *reinterpret_cast<const uint32_t*>(qin + g0 * d + c) : 0u;
        qa[dc][1] = g0 + 8 < G ? *reinterpret_cast<const uint32_t*>(qin + (g0 + 8) * d + c) : 0u;
        qa[dc][2] = g0 < G ? *reinterpret_cast<const uint32_t*>(qin + g0 * d + c + 8) : 0u;
        qa[dc][3] = g0 + 8 < G ? *reinterpret_cast<const uint32_t*>(qin + (g0 + 8) * d + c + 8) : 0u;
      }
    }
    const int m_ = lane >> 3, r_ = lane & 7;
    float mx0 = -INFINITY, mx1 = -INFINITY;
    bool aborted = false;
    // phase 1: logits
    for (int t = 0; t < nt; ++t) {
      const int st = t % kTcStages;
      if (!wait_bounded(&full[st], (t / kTcStages) & 1, gd)) {
        aborted = true;
        break;
      }
      const uint32_t tile = smem_u32(ring + st * tile_bytes);
      if (t == owner_tile && (next - j0 - t * kTcSlots) / 16 == warp) {
        const int r = next - j0 - t * kTcSlots;
        if (lane < d / 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kin + lane * 8);
          *reinterpret_cast<uint4*>(ring + (swz(tile, r, lane * 8) - smem_u32(ring))) = kv;
          reinterpret_cast<uint4*>(Kc + (long long)next * d)[lane] = kv;
          reinterpret_cast<uint4*>(Vc + (long long)next * d)[lane] = *reinterpret_cast<const uint4*>(vin + lane * 8);
        }
        if (lane == 0) pos[next] = pos_new;
        fence_proxy_async();
        __syncwarp();
      }
      float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int dc = 0; dc < 8; ++dc) {
        if (dc < ndc) {
          uint32_t b00, b01, b10, b11;
          ldsm_x4(swz(tile, warp * 16 + (m_ >> 1) * 8 + r_, dc * 16 + (m_ & 1) * 8), b00, b01, b10, b11);
          mma16816(d0, qa[dc], b00, b01);
          mma16816(d1, qa[dc], b10, b11);
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int jla = t * kTcSlots + warp * 16 + q4 * 2 + e;  // n-tile 0
        const int jlb = jla + 8;                                 // n-tile 1
        const float xa0 = jla < cnt ? d0[e] * a.scale2 : -INFINITY;
        const float xb0 = jlb < cnt ? d1[e] * a.scale2 : -INFINITY;
        const float xa1 = jla < cnt ? d0[2 + e] * a.scale2 : -INFINITY;
        const float xb1 = jlb < cnt ? d1[2 + e] * a.scale2 : -INFINITY;
        if (g0 < G) {
          xs[g0 * P.S_pad + jla] = xa0;
          xs[g0 * P.S_pad + jlb] = xb0;
          mx0 = fmaxf(mx0, fmaxf(xa0, xb0));
        }
        if (g0 + 8 < G) {
          xs[(g0 + 8) * P.S_pad + jla] = xa1;
          xs[(g0 + 8) * P.S_pad + jlb] = xb1;
          mx1 = fmaxf(mx1, fmaxf(xa1, xb1));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // phase 2: CTA max per query head
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (q4 == 0) {
      if (g0 < G) red_m[warp][g0] = mx0;
      if (g0 + 8 < G) red_m[warp][g0 + 8] = mx1;
    }
    named_bar_sync(1, kTcConsumers * 32);
    if (tid < G) {
      float v = -INFINITY;
      for (int w = 0; w < kTcConsumers; ++w) v = fmaxf(v, red_m[w][tid]);
      m_s[tid] = v;
    }
    named_bar_sync(1, kTcConsumers * 32);
    const float m0 = g0 < G ? m_s[g0] : 0.f;
    const float m1 = g0 + 8 < G ? m_s[g0 + 8] : 0.f;
    // phase 3: P V
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float l0 = 0.f, l1 = 0.f;
    for (int t = 0; t < nt && !aborted; ++t) {
      const int it = nt + t;
      const int st = it % kTcStages;
      if (!wait_bounded(&full[st], (it / kTcStages) & 1, gd)) {
        aborted = true;
        break;
      }
      const uint32_t tile = smem_u32(ring + st * tile_bytes);
      if (t == owner_tile && (next - j0 - t * kTcSlots) / 16 == warp) {
        const int r = next - j0 - t * kTcSlots;
        if (lane < d / 8)
          *reinterpret_cast<uint4*>(ring + (swz(tile, r, lane * 8) - smem_u32(ring))) =
              *reinterpret_cast<const uint4*>(vin + lane * 8);
        fence_proxy_async();
        __syncwarp();
      }
      const int jl = t * kTcSlots + warp * 16 + q4 * 2;
      uint32_t pa[4];
      {
        float p00 = 0.f, p01 = 0.f, p08 = 0.f, p09 = 0.f, p10 = 0.f, p11 = 0.f, p18 = 0.f, p19 = 0.f;
        if (g0 < G) {
          const float* xr = xs + g0 * P.S_pad + jl;
          p00 = ex2_approx(xr[0] - m0);
          p01 = ex2_approx(xr[1] - m0);
          p08 = ex2_approx(xr[8] - m0);
          p09 = ex2_approx(xr[9] - m0);
          l0 += (p00 + p01) + (p08 + p09);
        }
        if (g0 + 8 < G) {
          const float* xr = xs + (g0 + 8) * P.S_pad + jl;
          p10 = ex2_approx(xr[0] - m1);
          p11 = ex2_approx(xr[1] - m1);
          p18 = ex2_approx(xr[8] - m1);
          p19 = ex2_approx(xr[9] - m1);
          l1 += (p10 + p11) + (p18 + p19);
        }
        pa[0] = pack_bf16(p00, p01);
        pa[1] = pack_bf16(p10, p11);
        pa[2] = pack_bf16(p08, p09);
        pa[3] = pack_bf16(p18, p19);
      }
#pragma unroll
      for (int dn = 0; dn < 8; ++dn) {
        if (dn < ndc) {
          uint32_t b0a, b1a, b0b, b1b;
          ldsm_x4_t(swz(tile, warp * 16 + (m_ & 1) * 8 + r_, dn * 16 + (m_ >> 1) * 8), b0a, b1a, b0b, b1b);
          mma16816(o[2 * dn], pa, b0a, b1a);
          mma16816(o[2 * dn + 1], pa, b0b, b1b);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // CTA partials: O and row sums (shared-memory atomics across the 4 warps)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < 2 * ndc) {
        const int col = i * 8 + q4 * 2;
        if (g0 < G) {
          atomicAdd(&o_s[g0 * d + col], o[i][0]);
          atomicAdd(&o_s[g0 * d + col + 1], o[i][1]);
        }
        if (g0 + 8 < G) {
          atomicAdd(&o_s[(g0 + 8) * d + col], o[i][2]);
          atomicAdd(&o_s[(g0 + 8) * d + col + 1], o[i][3]);
        }
      }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    if (q4 == 0) {
      if (g0 < G) atomicAdd(&l_s[g0], l0);
      if (g0 + 8 < G) atomicAdd(&l_s[g0 + 8], l1);
    }
    if (aborted) abort_s = 1;
  }
  if (tid < G && cnt == 0) m_s[tid] = -INFINITY;
  __syncwarp();
  cluster.sync();

  // ---- combine over the cluster; each CTA writes a slice of the output
  if (tid < G * a.C) {
    const int r = tid / G, g = tid % G;
    mr_s[r][g] = *cluster.map_shared_rank(&m_s[g], r);
  }
  __syncthreads();
  if (tid < G) {
    float Mx = -INFINITY;
    for (int r = 0; r < a.C; ++r) Mx = fmaxf(Mx, mr_s[r][tid]);
    float Lsum = 0.f;
    for (int r = 0; r < a.C; ++r)
      if (mr_s[r][tid] > -INFINITY) Lsum += *cluster.map_shared_rank(&l_s[tid], r) * exp2f(mr_s[r][tid] - Mx);
    M_s[tid] = Mx;
    Li_s[tid] = Lsum > 0.f ? 1.f / Lsum : 0.f;
    lse_s[tid] = Mx + log2f(Lsum);
  }
  __syncthreads();
  {
    const int E = G * d;
    const int e0 = (int)((long long)E * rank / a.C), e1 = (int)((long long)E * (rank + 1) / a.C);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (long long)row * E;
    for (int i = e0 + tid; i < e1; i += kTcThreads) {
      const int g = i / d;
      float acc = 0.f;
      for (int r = 0; r < a.C; ++r) {
        const float mr = mr_s[r][g];
        if (mr > -INFINITY) acc += *cluster.map_shared_rank(&o_s[i], r) * exp2f(mr - M_s[g]);
      }
      out[i] = __float2bfloat16_rn(acc * Li_s[g]);
    }
  }

  // ---- exact probabilities into A, local eviction candidate
  Best best{INFINITY, -1, -1};
  if (ok && !abort_s) {
    int pos_thr;
    if (appended >= M) pos_thr = pos_new - M + 1;
    else pos_thr = pos[max(0, count0 - (M - appended))];
    for (int jl = tid; jl < cnt; jl += kTcThreads) {
      const int j = j0 + jl;
      float psum = 0.f;
      for (int g = 0; g < G; ++g) psum += ex2_approx(xs[g * P.S_pad + jl] - lse_s[g]);
      const float Anew = (j == next ? 0.f : a.gamma * A[j]) + psum;
      A[j] = Anew;
      const int pj = j == next ? pos_new : pos[j];
      if (j >= a.T && pj < pos_thr) {
        const Best c{Anew, pj, j};
        if (better(c, best)) best = c;
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
    for (int w = 1; w < kTcConsumers + 1; ++w)
      if (better(bw[w], bst)) bst = bw[w];
    best_s = bst;
  }
  __syncwarp();
  cluster.sync();

  if (rank == 0 && tid == 0 && ok) {
    Best bst = best_s;
    bool any_abort = abort_s != 0;
    for (int r = 1; r < a.C; ++r) {
      const Best y = *cluster.map_shared_rank(&best_s, r);
      if (better(y, bst)) bst = y;
      any_abort |= *cluster.map_shared_rank(&abort_s, r) != 0;
    }
    if (!any_abort) {
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
  }
  __syncwarp();
  cluster.sync();  // keep every CTA's shared memory alive until the others have read it
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

int launch_decode_init(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c,
                       cudaStream_t st) {
  (void)sh;
  decode_init_kernel<<<m.n_rows, 256, 0, st>>>(c.slot_off, c.b, p.sinks_T, p.recent_pct, c.A, c.meta, c.status);
  return cuda_status(cudaGetLastError());
}

int launch_decode(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c, const void* q_t,
                  const void* k_t, const void* v_t, void* out, cudaStream_t st) {
  if (sh.group > kMaxG) return KV_ERR_ARG;
  const int capb = cap_bound(sh, m, p);
  int C = 8;
  while (C > 1 && (capb + C - 1) / C < 128) C >>= 1;
  const int S_cap = (capb + C - 1) / C;
  DecArgs a;
  a.map = m;
  a.G = sh.group;
  a.d = sh.head_dim;
  a.C = C;
  a.S_cap = S_cap;
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

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(m.n_rows * C);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (sh.dtype == KV_BF16) {
    TcDec P;
    P.a = a;
    P.S_pad = ((S_cap + kTcSlots - 1) / kTcSlots) * kTcSlots + 4;
    P.nk = sh.head_dim / 64;
    P.limit_ns = kWaitLimitNs;
    const size_t smem = 1024 + (size_t)kTcStages * kTcSlots * sh.head_dim * 2 +
                        ((size_t)sh.group * P.S_pad + (size_t)sh.group * sh.head_dim) * sizeof(float);
    if (smem > 220 * 1024) return KV_ERR_ARG;
    const long long total = c.total_slots > 0 ? c.total_slots : kv_total_slots(&sh, m.L, m.n_seq, &p);
    CUtensorMap tmK, tmV;
    if (!encode_rows_bf16(&tmK, c.Kc, sh.head_dim, total, kTcSlots)) return KV_ERR_CUDA;
    if (!encode_rows_bf16(&tmV, c.Vc, sh.head_dim, total, kTcSlots)) return KV_ERR_CUDA;
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, tmK, tmV, P);
  } else {
    const size_t smem = ((size_t)sh.group * S_cap + 2 * (size_t)sh.group * sh.head_dim) * sizeof(float);
    if (smem > 200 * 1024) return KV_ERR_ARG;
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cudaFuncSetAttribute(decode_simple_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    e = cudaLaunchKernelEx(&cfg, decode_simple_kernel<float>, a);
  }
  return cuda_status(e);
}

}  // namespace kvc
