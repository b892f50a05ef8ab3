// kv_allocate: head-aware budget allocation (AudioKV blog §3.1, defaults in
// §5.1), one (sequence, layer) per warp (kv_allocate_global: one sequence per
// warp over all its layers' heads, with the layers' budgets pooled):
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

// One warp per allocation group: Hg heads sharing the budget of `layers`
// layers of one sequence (Hg = H, layers = 1: the per-layer allocation;
// Hg = n_layers H, layers = n_layers: one allocation over the sequence).
// Lanes take heads; sum S is added in head order by lane 0; the remainder goes
// to the heads ranked first by (fractional part descending, head ascending),
// the same set the one-at-a-time rule picks.
__global__ void allocate_kernel(const RowMap map, int Hg, int groups_per_seq, int layers, int H, int w, int pct,
                                double r, const float* __restrict__ S, int32_t* __restrict__ b) {
  extern __shared__ double xs[];  // [Hg]
  int* active = reinterpret_cast<int*>(xs + Hg);
  int* keep = active + Hg;
  __shared__ double sumS_s;
  const int lane = threadIdx.x;
  const int seq = blockIdx.x / groups_per_seq;
  const int grp = blockIdx.x % groups_per_seq;
  const long long L = map.L[seq];
  const float* Sg = S + (long long)grp * Hg;
  int32_t* bg = b + (long long)blockIdx.x * Hg;
  long long B_left = (long long)layers * (((long long)pct * L * H) / 100);
  int n_act = Hg;
  for (int h = lane; h < Hg; h += 32) active[h] = h;
  __syncwarp();
  for (;;) {
    if (n_act == 0) return;
    const long long B_rem = B_left - (long long)n_act * w;
    if (lane == 0) {
      double sumS = 0.0;
      for (int a = 0; a < n_act; ++a) sumS = __dadd_rn(sumS, (double)Sg[active[a]]);
      sumS_s = sumS;
    }
    __syncwarp();
    const double sumS = sumS_s;
    long long sum_b = 0;
    for (int a = lane; a < n_act; a += 32) {
      const int h = active[a];
      double x;
      if (sumS > 0.0) {
        double t1 = __dmul_rn(r, (double)B_rem);
        t1 = __ddiv_rn(t1, (double)n_act);
        double t2 = __dmul_rn(__dsub_rn(1.0, r), (double)B_rem);
        t2 = __dmul_rn(t2, (double)Sg[h]);
        t2 = __ddiv_rn(t2, sumS);
        x = __dadd_rn(__dadd_rn((double)w, t1), t2);
      } else {
        x = __dadd_rn((double)w, __ddiv_rn((double)B_rem, (double)n_act));
      }
      xs[a] = x;
      bg[h] = (int32_t)floor(x);
      sum_b += bg[h];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum_b += __shfl_xor_sync(0xffffffffu, sum_b, o);
    __syncwarp();
    const long long rem = B_left - sum_b;
    for (int a = lane; a < n_act; a += 32) {  // rank by (fractional part desc, head asc)
      const double f = __dsub_rn(xs[a], floor(xs[a]));
      int rank = 0;
      for (int a2 = 0; a2 < n_act; ++a2) {
        const double f2 = __dsub_rn(xs[a2], floor(xs[a2]));
        rank += f2 > f || (f2 == f && a2 < a);
      }
      if (rank < rem) bg[active[a]] += 1;
    }
    __syncwarp();
    // heads above L: capped, the rest re-allocated with what is left (in head order)
    bool capped = false;
    int n_keep = 0;
    long long B_cap = 0;
    for (int a0 = 0; a0 < n_act; a0 += 32) {
      const int a = a0 + lane;
      const int h = a < n_act ? active[a] : 0;
      const bool over = a < n_act && bg[h] > L;
      if (over) bg[h] = (int32_t)L;
      const unsigned bo = __ballot_sync(0xffffffffu, over);
      const unsigned bk = __ballot_sync(0xffffffffu, a < n_act && !over);
      if (a < n_act && !over) keep[n_keep + __popc(bk & ((1u << lane) - 1u))] = h;
      n_keep += __popc(bk);
      B_cap += (long long)__popc(bo) * L;
      capped = capped || bo != 0;
    }
    __syncwarp();
    if (!capped) return;
    B_left -= B_cap;
    for (int a = lane; a < n_keep; a += 32) active[a] = keep[a];
    n_act = n_keep;
    __syncwarp();
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
                    int64_t* slot_off, bool global, cudaStream_t st) {
  const int H = sh.n_kv_heads;
  const int Hg = global ? sh.n_layers * H : H;
  const int groups = global ? 1 : sh.n_layers;
  const size_t smem = (size_t)Hg * (sizeof(double) + 2 * sizeof(int));
  allocate_kernel<<<m.n_seq * groups, 32, smem, st>>>(m, Hg, groups, global ? sh.n_layers : 1, H, sh.w,
                                                      p.budget_pct, (double)p.r, S, b);
  slot_offsets_kernel<<<1, 1024, 0, st>>>(m.n_rows, b, slot_off);
  return cuda_status(cudaGetLastError());
}

}  // namespace kvc
