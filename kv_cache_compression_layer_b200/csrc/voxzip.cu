// kv_voxzip_pool: VoxZip's semantic-anchored pooling of the audio feature
// rows (VoxZip, 方法概述和架构, first stage).
//
// plan kernel (one CTA per sequence): every thread maps four segments'
// timestamps to row indices in float64; a block scan gives each kept
// segment the furthest end covered before it (its start is clipped to it)
// and the rows and groups of the segments before it, which place its groups
// and the copied gap in front of it in the output. Warps then write one
// (first row, row count, text row) descriptor per output row; the whole CTA
// writes the gap after the last segment.
//
// pool kernel (persistent, one wave of resident CTAs): a warp owns a 1 KB
// slice of one output row, reads the slice of each of the row's source rows
// with 16-byte loads (two rows, four pieces a lane, in flight), sums in
// float32 in row order, divides once, adds the text embedding and rounds
// once. Copied rows are exact.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "../../include/kvcomp_next.h"
#include "internal.h"

namespace kvc {
namespace {

struct VzMap {
  int n_seq;
  int L[KV_MAX_SEQ];
  int seg_off[KV_MAX_SEQ + 1];
  long long row_off[KV_MAX_SEQ + 1];
  double tau_total[KV_MAX_SEQ];
};

constexpr int kPlanThreads = 1024;
constexpr int kPlanPer = KV_VZ_MAX_SEGMENTS / kPlanThreads;  // segments per thread
static_assert(kPlanPer * kPlanThreads == KV_VZ_MAX_SEGMENTS, "segments per plan thread");

// floor(L tau / tau_total) clamped to [0, L]; the product rounds first.
__device__ __forceinline__ int vz_index(int L, double tau, double tau_total) {
  double x = floor(__ddiv_rn(__dmul_rn((double)L, tau), tau_total));
  x = fmin(fmax(x, 0.0), (double)L);
  return (int)x;
}

// Block-wide exclusive scan of (max, sum, sum) over threads in thread order;
// returns the block totals in tot_*.
__device__ void block_scan3(int vmax, int v1, int v2, int& ex_max, int& ex1, int& ex2, int& tot_max, int& tot1,
                            int& tot2, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int im = vmax, i1 = v1, i2 = v2;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int m = __shfl_up_sync(0xffffffffu, im, o), a = __shfl_up_sync(0xffffffffu, i1, o),
              b = __shfl_up_sync(0xffffffffu, i2, o);
    if (lane >= o) {
      im = max(im, m);
      i1 += a;
      i2 += b;
    }
  }
  if (lane == 31) {
    sh[warp] = im;
    sh[32 + warp] = i1;
    sh[64 + warp] = i2;
  }
  __syncthreads();
  if (warp == 0) {
    int wm = sh[lane], w1 = sh[32 + lane], w2 = sh[64 + lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int m = __shfl_up_sync(0xffffffffu, wm, o), a = __shfl_up_sync(0xffffffffu, w1, o),
                b = __shfl_up_sync(0xffffffffu, w2, o);
      if (lane >= o) {
        wm = max(wm, m);
        w1 += a;
        w2 += b;
      }
    }
    sh[96 + lane] = wm;
    sh[128 + lane] = w1;
    sh[160 + lane] = w2;
  }
  __syncthreads();
  const int pm = warp ? sh[96 + warp - 1] : 0, p1 = warp ? sh[128 + warp - 1] : 0, p2 = warp ? sh[160 + warp - 1] : 0;
  int wm = __shfl_up_sync(0xffffffffu, im, 1);  // exclusive max within the warp (values are >= 0)
  if (lane == 0) wm = 0;
  ex_max = max(pm, wm);
  ex1 = p1 + i1 - v1;
  ex2 = p2 + i2 - v2;
  tot_max = sh[96 + 31];
  tot1 = sh[128 + 31];
  tot2 = sh[160 + 31];
}

// Per-segment plan kept in shared memory between the scans and the writes.
struct SegPlan {
  int start;   // first covered row after clipping
  int len;     // rows pooled (0: the segment is not pooled)
  int groups;  // output rows of the segment
  int gap_lo;  // first row of the copied gap in front of it
  int shift;   // output row = feature row + shift, for the gap in front of it
  int text;    // text row of group 0, or -1 (no text add)
};

__global__ void __launch_bounds__(kPlanThreads)
    vz_plan_kernel(const VzMap m, float conf_min, const kv_asr_segment* __restrict__ segs, long long n_text_rows,
                   int has_text, int32_t* __restrict__ src, int32_t* __restrict__ out_len,
                   int32_t* __restrict__ status) {
  extern __shared__ SegPlan plan[];
  __shared__ int sh[192];
  const int s = blockIdx.x;
  const int L = m.L[s];
  const int n = m.seg_off[s + 1] - m.seg_off[s];
  const kv_asr_segment* sg = segs + m.seg_off[s];
  const double tt = m.tau_total[s];
  int32_t* out = src + 3 * m.row_off[s];

  // 1. timestamps -> rows; kept segments contribute their end to the coverage
  int a[kPlanPer], e[kPlanPer], nt[kPlanPer], tr[kPlanPer];
  bool keep[kPlanPer];
  int tmax = 0;
#pragma unroll
  for (int u = 0; u < kPlanPer; ++u) {
    const int i = threadIdx.x * kPlanPer + u;
    keep[u] = false;
    a[u] = e[u] = nt[u] = 0;
    tr[u] = -1;
    if (i < n) {
      const kv_asr_segment g = sg[i];
      a[u] = vz_index(L, g.tau_start, tt);
      e[u] = vz_index(L, g.tau_end, tt);
      nt[u] = g.n_text;
      tr[u] = g.text_row;
      keep[u] = g.confidence > conf_min && g.n_text >= 1 && e[u] > a[u];
      if (keep[u]) tmax = max(tmax, e[u]);
    }
  }
  int ex_max, ex1, ex2, cover, t1, t2;
  block_scan3(tmax, 0, 0, ex_max, ex1, ex2, cover, t1, t2, sh);
  // 2. clipped starts, pooled rows and groups of each segment
  int len[kPlanPer], grp[kPlanPer], prev[kPlanPer];
  int run = ex_max, tlen = 0, tgrp = 0;
#pragma unroll
  for (int u = 0; u < kPlanPer; ++u) {
    prev[u] = run;
    const int st = max(a[u], run);
    len[u] = keep[u] ? max(0, e[u] - st) : 0;
    grp[u] = len[u] > 0 ? min(nt[u], len[u]) : 0;
    a[u] = st;
    if (keep[u]) run = max(run, e[u]);
    tlen += len[u];
    tgrp += grp[u];
  }
  __syncthreads();  // sh is reused by the second scan
  int tot_len, tot_grp, unused;
  block_scan3(0, tlen, tgrp, ex_max, ex1, ex2, unused, tot_len, tot_grp, sh);
  int cl = ex1, cg = ex2;
#pragma unroll
  for (int u = 0; u < kPlanPer; ++u) {
    const int i = threadIdx.x * kPlanPer + u;
    if (i < n) {
      int text = tr[u];
      if (has_text && len[u] > 0 && (text < 0 || (long long)text + grp[u] > n_text_rows)) {
        atomicOr(status, KV_DEV_RANGE);
        text = -1;
      }
      plan[i] = SegPlan{a[u], len[u], grp[u], prev[u], cg - cl, text};
    }
    cl += len[u];
    cg += grp[u];
  }
  if (threadIdx.x == 0) out_len[s] = L - tot_len + tot_grp;
  __syncthreads();

  // 3. descriptors: a warp per segment (its gap, then its groups); the CTA
  // writes the gap after the furthest covered row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = warp; i < n; i += kPlanThreads / 32) {
    const SegPlan p = plan[i];
    if (p.len == 0) continue;
    for (int t = p.gap_lo + lane; t < p.start; t += 32) {
      const int r = t + p.shift;
      out[3 * r] = t;
      out[3 * r + 1] = 1;
      out[3 * r + 2] = -1;
    }
    const int r0 = p.start + p.shift;
    for (int j = lane; j < p.groups; j += 32) {
      const int lo = (int)((long long)j * p.len / p.groups), hi = (int)((long long)(j + 1) * p.len / p.groups);
      const int r = r0 + j;
      out[3 * r] = p.start + lo;
      out[3 * r + 1] = hi - lo;
      out[3 * r + 2] = has_text && p.text < 0 ? -1 : p.text + j;
    }
  }
  const int tail_shift = tot_grp - tot_len;
  for (int t = cover + threadIdx.x; t < L; t += kPlanThreads) {
    const int r = t + tail_shift;
    out[3 * r] = t;
    out[3 * r + 1] = 1;
    out[3 * r + 2] = -1;
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(float* acc, const uint4& v) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
  __device__ static uint4 pack(const float* x) {
    uint4 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    return r;
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void add(float* acc, const uint4& v) {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float* x) {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
  }
};

constexpr int kPoolThreads = 256;
constexpr int kSliceBytes = 1024;  // a warp's share of a row: two 16-byte pieces per lane

template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
    vz_pool_kernel(const VzMap m, int d, int slices, long long units, const T* __restrict__ E_A,
                   const T* __restrict__ E_T, int has_text, T* __restrict__ E_comp, const int32_t* __restrict__ src,
                   const int32_t* __restrict__ out_len) {
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * kPoolThreads) >> 5;
  for (long long u = ((long long)blockIdx.x * kPoolThreads + threadIdx.x) >> 5; u < units; u += nw) {
    const long long R = u / slices;
    const int slice = (int)(u - R * slices);
    int lo_s = 0, hi_s = m.n_seq - 1;  // the sequence whose rows hold R
    while (lo_s < hi_s) {
      const int mid = (lo_s + hi_s + 1) >> 1;
      if (m.row_off[mid] <= R) lo_s = mid;
      else hi_s = mid - 1;
    }
    const long long r = R - m.row_off[lo_s];
    if (r >= __ldg(out_len + lo_s)) continue;
    const int first = __ldg(src + 3 * R), cnt = __ldg(src + 3 * R + 1), tr = __ldg(src + 3 * R + 2);
    if (!kv_check(first >= 0 && cnt >= 0 && (long long)first + cnt <= m.L[lo_s])) continue;
    const int c0 = slice * (kSliceBytes / (int)sizeof(T)) + lane * N;  // first piece
    const int c1 = c0 + 32 * N;                                        // second piece
    const bool p0 = c0 < d, p1 = c1 < d;
    const T* base = E_A + (m.row_off[lo_s] + first) * (long long)d;
    float acc0[N], acc1[N];
#pragma unroll
    for (int i = 0; i < N; ++i) acc0[i] = acc1[i] = 0.f;
    int k = 0;
    for (; k + 2 <= cnt; k += 2) {  // two source rows (four pieces) in flight
      uint4 x00 = {}, x01 = {}, x10 = {}, x11 = {};
      if (p0) {
        x00 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)k * d + c0));
        x10 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)(k + 1) * d + c0));
      }
      if (p1) {
        x01 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)k * d + c1));
        x11 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)(k + 1) * d + c1));
      }
      Vec<T>::add(acc0, x00);
      Vec<T>::add(acc1, x01);
      Vec<T>::add(acc0, x10);
      Vec<T>::add(acc1, x11);
    }
    if (k < cnt) {
      uint4 x0 = {}, x1 = {};
      if (p0) x0 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)k * d + c0));
      if (p1) x1 = __ldcs(reinterpret_cast<const uint4*>(base + (long long)k * d + c1));
      Vec<T>::add(acc0, x0);
      Vec<T>::add(acc1, x1);
    }
    if (cnt != 1) {
      const float fc = (float)cnt;
#pragma unroll
      for (int i = 0; i < N; ++i) {
        acc0[i] = __fdiv_rn(acc0[i], fc);
        acc1[i] = __fdiv_rn(acc1[i], fc);
      }
    }
    if (has_text && tr >= 0) {
      float t0[N], t1[N];
#pragma unroll
      for (int i = 0; i < N; ++i) t0[i] = t1[i] = 0.f;
      const T* trow = E_T + (long long)tr * d;
      if (p0) Vec<T>::add(t0, __ldg(reinterpret_cast<const uint4*>(trow + c0)));
      if (p1) Vec<T>::add(t1, __ldg(reinterpret_cast<const uint4*>(trow + c1)));
#pragma unroll
      for (int i = 0; i < N; ++i) {
        acc0[i] += t0[i];
        acc1[i] += t1[i];
      }
    }
    T* orow = E_comp + R * (long long)d;
    if (p0) __stcs(reinterpret_cast<uint4*>(orow + c0), Vec<T>::pack(acc0));
    if (p1) __stcs(reinterpret_cast<uint4*>(orow + c1), Vec<T>::pack(acc1));
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" int kv_voxzip_pool(const int32_t* L_a, int32_t n_seq, const double* tau_total, const int32_t* seg_off,
                              int32_t d, int32_t dtype, float conf_min, const kv_asr_segment* segs, const void* E_A,
                              const void* E_T, int64_t n_text_rows, void* E_comp, int32_t* src, int32_t* out_len,
                              int32_t* status, void* stream) {
  if (!L_a || !tau_total || !seg_off || n_seq < 1 || n_seq > KV_MAX_SEQ) return KV_ERR_ARG;
  if (dtype != KV_BF16 && dtype != KV_F32) return KV_ERR_ARG;
  const int esz = dtype == KV_BF16 ? 2 : 4;
  if (d < 1 || d > KV_VZ_MAX_D || (d * esz) % 16) return KV_ERR_ARG;
  if (!E_A || !E_comp || !src || !out_len || !aligned16(E_A) || !aligned16(E_comp)) return KV_ERR_ARG;
  if (E_T && (!aligned16(E_T) || n_text_rows < 0)) return KV_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(src) & 3u) || (reinterpret_cast<uintptr_t>(out_len) & 3u)) return KV_ERR_ARG;
  if (E_T && !status) return KV_ERR_ARG;  // a text row out of range needs somewhere to be reported
  VzMap m;
  std::memset(&m, 0, sizeof(m));
  m.n_seq = n_seq;
  if (seg_off[0] != 0) return KV_ERR_ARG;
  long long rows = 0;
  int max_seg = 0;
  for (int s = 0; s < n_seq; ++s) {
    if (L_a[s] < 1 || L_a[s] > KV_VZ_MAX_L) return KV_ERR_ARG;
    if (!(tau_total[s] > 0.0) || !std::isfinite(tau_total[s])) return KV_ERR_ARG;
    const int ns = seg_off[s + 1] - seg_off[s];
    if (ns < 0 || ns > KV_VZ_MAX_SEGMENTS) return KV_ERR_ARG;
    max_seg = std::max(max_seg, ns);
    m.L[s] = L_a[s];
    m.seg_off[s] = seg_off[s];
    m.row_off[s] = rows;
    m.tau_total[s] = tau_total[s];
    rows += L_a[s];
  }
  m.seg_off[n_seq] = seg_off[n_seq];
  m.row_off[n_seq] = rows;
  if (rows >= (1ll << 31)) return KV_ERR_ARG;
  if (seg_off[n_seq] > 0 && (!segs || (reinterpret_cast<uintptr_t>(segs) & 7u))) return KV_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  const size_t plan_bytes = sizeof(SegPlan) * (size_t)std::max(max_seg, 1);
  // a per-device setting: made on every launch (cheap), for whichever device is current
  if (cudaFuncSetAttribute(vz_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(sizeof(SegPlan) * KV_VZ_MAX_SEGMENTS)) != cudaSuccess)
    return KV_ERR_CUDA;
  vz_plan_kernel<<<n_seq, kPlanThreads, plan_bytes, st>>>(m, conf_min, segs, (long long)n_text_rows,
                                                          E_T ? 1 : 0, src, out_len, status);
  const int slices = (d * esz + kSliceBytes - 1) / kSliceBytes;
  const long long units = rows * slices;
  const long long want = (units * 32 + kPoolThreads - 1) / kPoolThreads;
  // one wave: as many CTAs as are resident at once (no tail of late CTAs)
  auto grid_of = [&](const void* kernel) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kPoolThreads, 0);
    return (int)std::max(1ll, std::min<long long>(want, (long long)sm_count() * std::max(1, per_sm)));
  };
  if (dtype == KV_BF16)
    vz_pool_kernel<__nv_bfloat16><<<grid_of((const void*)vz_pool_kernel<__nv_bfloat16>), kPoolThreads, 0, st>>>(
        m, d, slices, units, static_cast<const __nv_bfloat16*>(E_A), static_cast<const __nv_bfloat16*>(E_T),
        E_T ? 1 : 0, static_cast<__nv_bfloat16*>(E_comp), src, out_len);
  else
    vz_pool_kernel<float><<<grid_of((const void*)vz_pool_kernel<float>), kPoolThreads, 0, st>>>(
        m, d, slices, units, static_cast<const float*>(E_A), static_cast<const float*>(E_T), E_T ? 1 : 0,
        static_cast<float*>(E_comp), src, out_len);
  return cuda_status(cudaGetLastError());
}
