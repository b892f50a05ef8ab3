// kv_select_gather: per-row top-k selection and compaction of the kept K/V
// (AudioKV blog §3.1: a basic local window is always kept, the rest of the
// row's budget goes to the highest smoothed scores; the C3 page's bypass keeps
// every position once the budget reaches the audio length).
//
// select kernel (one CTA per row; in the WnW segment-wise variant each warp
// takes whole segments, so the row's segments are selected in parallel):
// smoothed scores become order-preserving
// uint32 keys (-0 folded into +0) in shared memory; an MSB-first 8-bit radix
// select finds the k-th largest key T and how many keys equal to T are taken;
// a warp-ballot compaction then writes the kept indices in ascending order:
// keys above T, the first (k - #above) keys equal to T, and the window.
//
// gather kernel (persistent, all SMs): warps walk the compacted slots in
// units of 32, and copy each kept K and V row with 16-byte loads/stores.
#include "internal.h"

namespace kvc {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

__host__ __device__ __forceinline__ int map_max_len(const RowMap& m) {
  int x = 0;
  for (int i = 0; i < m.n_seq; ++i) x = m.L[i] > x ? m.L[i] : x;
  return x;
}

// Dynamic shared memory of select_kernel: the keys of the longest row, for the
// segment-wise variant the quotas and their prefix, and the warps' histograms.
size_t sel_smem_bytes(const RowMap& m, int nseg) {
  size_t b = (size_t)map_max_len(m) * sizeof(uint32_t);
  if (nseg > 0) b += 2 * (size_t)nseg * sizeof(int);
  return b + (size_t)kSelWarps * 256 * sizeof(int);
}

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The k largest keys of keys[c0s, c1s) (ties to the lower index) written to
// out[0, k) in ascending index order; called by the whole block. Each radix
// round counts into per-warp histograms (no atomics between warps: the
// scores' top bytes take few values), merged once per round.
__device__ void select_range(const uint32_t* keys, int c0s, int c1s, int k, int32_t* __restrict__ out, int* hist,
                             int (*whist)[256], int* wgt, int* weq, uint32_t* sh_prefix, int* sh_kk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = c1s - c0s;
  __syncthreads();  // the keys are in place, the previous range's scratch is free
  if (threadIdx.x == 0) {
    *sh_prefix = 0;
    *sh_kk = k;
  }
  __syncthreads();
  // radix select of the k-th largest key, most significant byte first
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < kSelWarps * 256; i += kSelThreads) (&whist[0][0])[i] = 0;
    __syncthreads();
    const uint32_t prefix = *sh_prefix;
    for (int j = c0s + threadIdx.x; j < c1s; j += kSelThreads) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += kSelThreads) {  // warp order: a fixed sum
      int t = 0;
      for (int w = 0; w < kSelWarps; ++w) t += whist[w][b];
      hist[b] = t;
    }
    __syncthreads();
    if (warp == 0) {
      int kk = *sh_kk;
      const int dg = top_bin(hist, kk);
      if (lane == 0) {
        *sh_kk = kk;
        *sh_prefix = prefix | ((uint32_t)dg << shift);
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = *sh_prefix;
  const int take_eq = *sh_kk;  // keys equal to T to keep, lowest indices first

  // per-warp counts over contiguous chunks, then ballot compaction in index order
  const int chunk = (((n + kSelWarps - 1) / kSelWarps) + 31) & ~31;
  const int c0 = c0s + warp * chunk, c1 = min(c1s, c0 + chunk);
  int ngt = 0, neq = 0;
  for (int j = c0 + lane; j < c1; j += 32) {
    const uint32_t key = keys[j];
    ngt += key > T;
    neq += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
    neq += __shfl_xor_sync(0xffffffffu, neq, o);
  }
  if (lane == 0) {
    wgt[warp] = ngt;
    weq[warp] = neq;
  }
  __syncthreads();
  int eq_before = 0, sel_before = 0;
  for (int i = 0; i < warp; ++i) {
    sel_before += wgt[i] + max(0, min(weq[i], take_eq - eq_before));
    eq_before += weq[i];
  }
  const unsigned lt = (1u << lane) - 1u;
  for (int base = c0; base < c1; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < c1 ? keys[j] : 0u;
    const bool eq = j < c1 && key == T;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_before + __popc(beq & lt);
    const bool sel = j < c1 && (key > T || (eq && eq_rank < take_eq));
    const unsigned bsel = __ballot_sync(0xffffffffu, sel);
    const int at = sel_before + __popc(bsel & lt);
    if (sel && at < k) out[at] = j;
    eq_before += __popc(beq);
    sel_before += __popc(bsel);
  }
}

// The same selection by one warp (a segment of the segment-wise variant):
// keys[c0, c1) -> out[0, k), 1 <= k <= c1 - c0; hist is the warp's 256 bins.
__device__ void select_range_warp(const uint32_t* keys, int c0, int c1, int k, int32_t* __restrict__ out,
                                  int* hist) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hist[i] = 0;
    __syncwarp();
    for (int j = c0 + lane; j < c1; j += 32) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    const int dg = top_bin(hist, kk);
    prefix |= (uint32_t)dg << shift;
    mask |= 255u << shift;
    __syncwarp();  // every lane has read the bins before the next round clears them
  }
  const uint32_t T = prefix;
  const int take_eq = kk;
  const unsigned lt = (1u << lane) - 1u;
  int eq_before = 0, sel_before = 0;
  for (int base = c0; base < c1; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < c1 ? keys[j] : 0u;
    const bool eq = j < c1 && key == T;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const bool sel = j < c1 && (key > T || (eq && eq_before + __popc(beq & lt) < take_eq));
    const unsigned bsel = __ballot_sync(0xffffffffu, sel);
    const int at = sel_before + __popc(bsel & lt);
    if (sel && at < k) out[at] = j;
    eq_before += __popc(beq);
    sel_before += __popc(bsel);
  }
}

// One CTA per row. nseg = 0: one top-(b - w) over the candidates [0, L - w);
// nseg > 0: the candidates cut into nseg segments [floor(i n / nseg),
// floor((i + 1) n / nseg)), segment i keeping q_i = floor(k len_i / n) plus
// one for the (k - sum q) largest remainders k len_i mod n (ties to the lower
// segment) -- WnW's segment-wise static subset.
__global__ void __launch_bounds__(kSelThreads, 1)
    select_kernel(const RowMap map, int w, int nseg, const float* __restrict__ s_hat, const int32_t* __restrict__ b,
                  const int64_t* __restrict__ slot_off, int32_t* __restrict__ idx) {
  // dynamic shared memory: keys [L]; with segments also q_s, at_s [nseg] and
  // the warps' histograms [kSelWarps][256] (sel_smem_bytes)
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int wgt[kSelWarps], weq[kSelWarps];
  __shared__ uint32_t sh_prefix;
  __shared__ int sh_kk;

  const int row = blockIdx.x;
  int* q_s = reinterpret_cast<int*>(keys + map_max_len(map));
  int* at_s = q_s + max(nseg, 0);
  int(*whist)[256] = reinterpret_cast<int(*)[256]>(at_s + max(nseg, 0));
  const int L = row_len(map, row);
  const long long koff = row_key_off(map, row);
  const int bb = b[row];
  int32_t* out = idx + slot_off[row];
  // debug builds: the row writes min(b, L) entries into its b + 1 slots
  if (!kv_check(bb < 0 || min(bb, L) <= slot_off[row + 1] - slot_off[row])) return;

  if (bb >= L) {
    for (int j = threadIdx.x; j < L; j += kSelThreads) out[j] = j;
    return;
  }
  if (bb < w) return;  // not a valid budget (kv_allocate never produces one); nothing is written
  const int n = L - w;  // candidates [0, n); the window [n, L) is always kept
  const int k = bb - w;
  for (int i = threadIdx.x; i < w; i += kSelThreads) out[k + i] = n + i;
  if (k <= 0) return;
  for (int j = threadIdx.x; j < n; j += kSelThreads) keys[j] = order_key(s_hat[koff + j]);
  if (nseg <= 1) {  // one top-k over the candidates (a single segment is the same selection)
    select_range(keys, 0, n, k, out, hist, whist, wgt, weq, &sh_prefix, &sh_kk);
    return;
  }
  // segment quotas: q_i = floor(k len_i / n), the remainder by largest k len_i mod n
  for (int i = threadIdx.x; i < nseg; i += kSelThreads) {
    const long long len = (long long)(i + 1) * n / nseg - (long long)i * n / nseg;
    const long long fr = (long long)k * len % n;
    long long sum_q = 0;
    int rank = 0;
    for (int i2 = 0; i2 < nseg; ++i2) {
      const long long len2 = (long long)(i2 + 1) * n / nseg - (long long)i2 * n / nseg;
      sum_q += (long long)k * len2 / n;
      const long long fr2 = (long long)k * len2 % n;
      rank += fr2 > fr || (fr2 == fr && i2 < i);
    }
    q_s[i] = (int)((long long)k * len / n) + (rank < k - sum_q ? 1 : 0);
  }
  __syncthreads();
  // each segment's first output place: the exclusive prefix of the quotas
  // (each thread sums a run of consecutive segments, then the runs are scanned)
  {
    const int per = (nseg + kSelThreads - 1) / kSelThreads;
    const int i0 = threadIdx.x * per, i1 = min(nseg, i0 + per);
    int run = 0;
    for (int i = i0; i < i1; ++i) run += q_s[i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wgt[warp] = incl;
    __syncthreads();
    int before = incl - run;
    for (int i = 0; i < warp; ++i) before += wgt[i];
    for (int i = i0; i < i1; ++i) {
      at_s[i] = before;
      before += q_s[i];
    }
  }
  __syncthreads();
  if (nseg < kSelWarps / 4) {  // a few long segments: the whole block on each in turn
    for (int i = 0; i < nseg; ++i) {
      const int lo = (int)((long long)i * n / nseg), hi = (int)((long long)(i + 1) * n / nseg);
      if (q_s[i] > 0) select_range(keys, lo, hi, q_s[i], out + at_s[i], hist, whist, wgt, weq, &sh_prefix, &sh_kk);
    }
    return;
  }
  // many segments: one warp each, in parallel
  const int warp = threadIdx.x >> 5;
  for (int i = warp; i < nseg; i += kSelWarps) {
    const int lo = (int)((long long)i * n / nseg), hi = (int)((long long)(i + 1) * n / nseg);
    const int q = q_s[i];
    if (q > 0) select_range_warp(keys, lo, hi, q, out + at_s[i], whist[warp]);
  }
}

__global__ void __launch_bounds__(256)
    gather_kernel(const RowMap map, int row_bytes, const int64_t* __restrict__ slot_off,
                  const int32_t* __restrict__ b, const int32_t* __restrict__ idx, const uint8_t* __restrict__ K,
                  const uint8_t* __restrict__ V, uint8_t* __restrict__ Kc, uint8_t* __restrict__ Vc) {
  const int n_rows = map.n_rows;
  const long long total = slot_off[n_rows];
  const int lane = threadIdx.x & 31;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int chunks = row_bytes / 16;       // 16-byte pieces per K/V row
  const int per_iter = max(1, 32 / chunks);  // rows copied per warp instruction
  for (long long unit = gw; unit * 32 < total; unit += nw) {
    const long long slot = unit * 32 + lane;
    long long src = -1;
    if (slot < total) {
      int lo = 0, hi = n_rows - 1;  // last row with slot_off[row] <= slot
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (slot_off[mid] <= slot) lo = mid;
        else hi = mid - 1;
      }
      const long long t = slot - slot_off[lo];
      if (t < b[lo]) {
        const int j = idx[slot];
        if (j >= 0 && j < row_len(map, lo)) src = row_key_off(map, lo) + j;  // skips rows select left unwritten
      }
    }
    for (int i0 = 0; i0 < 32; i0 += per_iter) {
      const int i = i0 + (per_iter > 1 ? lane / chunks : 0);
      const long long sidx = __shfl_sync(0xffffffffu, src, min(i, 31));
      const int piece = per_iter > 1 ? lane % chunks : lane;
      if (i < 32 && sidx >= 0) {
        const long long dst = unit * 32 + i;
        for (int c = piece; c < chunks; c += 32) {
          const uint4 kv = __ldg(reinterpret_cast<const uint4*>(K + sidx * row_bytes) + c);
          const uint4 vv = __ldg(reinterpret_cast<const uint4*>(V + sidx * row_bytes) + c);
          reinterpret_cast<uint4*>(Kc + dst * row_bytes)[c] = kv;
          reinterpret_cast<uint4*>(Vc + dst * row_bytes)[c] = vv;
        }
      }
    }
  }
}

}  // namespace

int launch_select_gather(const kv_shape& sh, const RowMap& m, const float* s_hat, const void* K, const void* V,
                         const int32_t* b, const int64_t* slot_off, int32_t* idx, void* Kc, void* Vc, int nseg,
                         cudaStream_t st) {
  // a per-device setting: made on every launch (cheap), for whichever device is current
  const size_t smem = sel_smem_bytes(m, nseg);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return KV_ERR_CUDA;
  select_kernel<<<m.n_rows, kSelThreads, smem, st>>>(m, sh.w, nseg, s_hat, b, slot_off, idx);
  const int esz = sh.dtype == KV_BF16 ? 2 : 4;
  const int row_bytes = sh.head_dim * esz;
  gather_kernel<<<sm_count() * 8, 256, 0, st>>>(m, row_bytes, slot_off, b, idx, static_cast<const uint8_t*>(K),
                                               static_cast<const uint8_t*>(V), static_cast<uint8_t*>(Kc),
                                               static_cast<uint8_t*>(Vc));
  return cuda_status(cudaGetLastError());
}

}  // namespace kvc
