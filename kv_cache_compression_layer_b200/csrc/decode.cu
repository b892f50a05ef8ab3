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

#include "decode_common.cuh"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& y, float x) { y = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& y, float x) { y = __float2bfloat16_rn(x); }

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
  const bool ok = S <= a.S_cap && count < cap && (!evict || bb >= a.T + M) && kv_check(next >= 0 && next < cap);
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
    // the warps add their partials in warp order: a fixed summation order, so a
    // step's result does not depend on scheduling
    for (int w = 0; w < kDecWarps; ++w) {
      if (warp == w) {
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < per) o_s[g * d + lane * per + e] += acc[g][e];
      }
      __syncthreads();
    }
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
    int pos_thr = pos_new - M + 1;
    if (appended < M && kv_check(count0 - (M - appended) < cap)) pos_thr = pos[max(0, count0 - (M - appended))];
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
    if (evict && bst.slot >= 0 && kv_check(bst.slot < cap)) {
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

// Largest b_i + 1 a row can have: b_h <= min(L, B - (H' - 1) w) since every
// other head sharing the budget B keeps at least w (H' = H heads of a layer,
// or all n_layers H heads of a sequence for kv_allocate_global).
int cap_bound(const kv_shape& sh, const RowMap& m, const kv_params& p) {
  long long mx = 0;
  for (int s = 0; s < m.n_seq; ++s) {
    const long long L = m.L[s];
    // the larger of the per-layer and the pooled (kv_allocate_global) bounds
    const long long B = (long long)sh.n_layers * (((long long)p.budget_pct * L * sh.n_kv_heads) / 100);
    const long long bmax = std::min(L, B - ((long long)sh.n_layers * sh.n_kv_heads - 1) * sh.w);
    mx = std::max(mx, bmax + 1);
  }
  return (int)mx;
}

}  // namespace

int cap_bound_of(const kv_shape& sh, const RowMap& m, const kv_params& p) { return cap_bound(sh, m, p); }

static bool tc_path(const kv_shape& sh) { return sh.dtype == KV_BF16 && sh.group <= kTcMaxG; }

size_t decode_scratch_bytes(const kv_shape& sh, const RowMap& m, const kv_params& p, long long total_slots) {
  return tc_path(sh) ? tc_scratch_bytes(sh, m, cap_bound(sh, m, p), total_slots) : 0;
}

static long long cache_slots(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c) {
  return c.total_slots > 0 ? c.total_slots : kv_total_slots(&sh, m.L, m.n_seq, &p);
}

int launch_decode_init(const kv_shape& sh, const RowMap& m, const kv_params& p, const kv_cache& c,
                       cudaStream_t st) {
  decode_init_kernel<<<m.n_rows, 256, 0, st>>>(c.slot_off, c.b, p.sinks_T, p.recent_pct, c.A, c.meta, c.status);
  if (tc_path(sh)) return launch_tc_init(sh, m, cap_bound(sh, m, p), cache_slots(sh, m, p, c), c, st);
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
  if (tc_path(sh)) {
    a.C = 1;
    a.S_cap = 0;
    return launch_tc(sh, m, capb, cache_slots(sh, m, p, c), a, c, st);
  }
  cudaError_t e;
  {
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
      e = cudaFuncSetAttribute(decode_simple_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               200 * 1024);
      if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, decode_simple_kernel<__nv_bfloat16>, a);
    } else {
      e = cudaFuncSetAttribute(decode_simple_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, decode_simple_kernel<float>, a);
    }
  }
  return cuda_status(e);
}

}  // namespace kvc
