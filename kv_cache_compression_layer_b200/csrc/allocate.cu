// kv_allocate: head-aware budget allocation (AudioKV blog §3.1, defaults in
// §5.1), one (sequence, layer) per block:
//   B = floor(pct L H / 100),  B_rem = B - H w,
//   x_h = w + r B_rem / H + (1 - r) B_rem S_h / sum_h S_h,
//   b_h = floor(x_h), the remainder +1 to the largest fractional parts (ties
//   to the lower head); heads above L are capped at L and the remaining
//   heads re-allocated with what is left; sum S = 0 splits evenly.
// The arithmetic is float64 with explicitly rounded operations in a fixed
// order (no contraction into FMA), so the result is reproducible bit for bit:
//   t1 = r*B_rem; t1 = t1/H; t2 = (1-r)*B_rem; t2 = t2*S_h; t2 = t2/sumS;
//   x = (w + t1) + t2.
// A second kernel writes slot_off, the prefix of b_i + 1 over rows (each row
// keeps one spare slot for the token a decode step appends).
#include "internal.h"

namespace kvc {
namespace {

__global__ void allocate_kernel(const RowMap map, int H, int w, int pct, double r, const float* __restrict__ S,
                                int32_t* __restrict__ b) {
  extern __shared__ double xs[];  // [H]
  int* active = reinterpret_cast<int*>(xs + H);
  int* keep = active + H;
  int* taken = keep + H;
  if (threadIdx.x != 0) return;
  const int seq = blockIdx.x / (map.rows_per_seq / H);
  const int layer = blockIdx.x % (map.rows_per_seq / H);
  const long long L = map.L[seq];
  const float* Sl = S + (long long)layer * H;
  int32_t* bl = b + (long long)blockIdx.x * H;
  long long B_left = ((long long)pct * L * H) / 100;
  int n_act = H;
  for (int h = 0; h < H; ++h) active[h] = h;
  for (;;) {
    if (n_act == 0) return;
    const long long B_rem = B_left - (long long)n_act * w;
    double sumS = 0.0;
    for (int a = 0; a < n_act; ++a) sumS = __dadd_rn(sumS, (double)Sl[active[a]]);
    long long sum_b = 0;
    for (int a = 0; a < n_act; ++a) {
      const int h = active[a];
      double x;
      if (sumS > 0.0) {
        double t1 = __dmul_rn(r, (double)B_rem);
        t1 = __ddiv_rn(t1, (double)n_act);
        double t2 = __dmul_rn(__dsub_rn(1.0, r), (double)B_rem);
        t2 = __dmul_rn(t2, (double)Sl[h]);
        t2 = __ddiv_rn(t2, sumS);
        x = __dadd_rn(__dadd_rn((double)w, t1), t2);
      } else {
        x = __dadd_rn((double)w, __ddiv_rn((double)B_rem, (double)n_act));
      }
      xs[a] = x;
      bl[h] = (int32_t)floor(x);
      sum_b += bl[h];
      taken[a] = 0;
    }
    const long long rem = B_left - sum_b;
    for (long long k = 0; k < rem; ++k) {
      int best = -1;
      double bf = -1.0;
      for (int a = 0; a < n_act; ++a) {
        if (taken[a]) continue;
        const double f = __dsub_rn(xs[a], floor(xs[a]));
        if (f > bf) {
          bf = f;
          best = a;
        }
      }
      if (best < 0) break;
      taken[best] = 1;
      bl[active[best]] += 1;
    }
    bool capped = false;
    int n_keep = 0;
    for (int a = 0; a < n_act; ++a) {
      const int h = active[a];
      if (bl[h] > L) {
        bl[h] = (int32_t)L;
        B_left -= L;
        capped = true;
      } else {
        keep[n_keep++] = h;
      }
    }
    if (!capped) return;
    for (int a = 0; a < n_keep; ++a) active[a] = keep[a];
    n_act = n_keep;
  }
}

// slot_off[i] = sum_{i' < i} (b_i' + 1), one block.
__global__ void slot_offsets_kernel(int n_rows, const int32_t* __restrict__ b, int64_t* __restrict__ slot_off) {
  __shared__ long long warp_tot[32];
  __shared__ long long carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_rows; base += blockDim.x) {
    const int i = base + threadIdx.x;
    long long v = i < n_rows ? (long long)b[i] + 1 : 0;
    // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    long long wbefore = 0;
    for (int k = 0; k < warp; ++k) wbefore += warp_tot[k];
    const long long incl = carry + wbefore + v;
    const long long own = i < n_rows ? (long long)b[i] + 1 : 0;
    if (i < n_rows) slot_off[i] = incl - own;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) slot_off[n_rows] = carry;
}

}  // namespace

int launch_allocate(const kv_shape& sh, const RowMap& m, const kv_params& p, const float* S, int32_t* b,
                    int64_t* slot_off, cudaStream_t st) {
  const int H = sh.n_kv_heads;
  const size_t smem = (size_t)H * (sizeof(double) + 3 * sizeof(int));
  allocate_kernel<<<m.n_seq * sh.n_layers, 32, smem, st>>>(m, H, sh.w, p.budget_pct, (double)p.r, S, b);
  slot_offsets_kernel<<<1, 1024, 0, st>>>(m.n_rows, b, slot_off);
  return cuda_status(cudaGetLastError());
}

}  // namespace kvc
