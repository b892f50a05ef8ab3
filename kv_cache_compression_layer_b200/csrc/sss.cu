// kv_sss: Spectral Score Smoothing (AudioKV blog §2.2), one row per CTA
// cluster.
//
//   F = RFFT(s);  E(k) = sum_{i<=k} |F_i|^2;  k* = min{k : E(k) >= rho E(L/2)};
//   s_hat = (1 - alpha) s + alpha IRFFT(F 1[i <= k*], n = L).
//
// The real row of even length L is packed as N = L/2 complex points
// z_m = s_{2m} + i s_{2m+1} and transformed in shared memory by a Stockham
// (self-sorting) mixed-radix FFT with radices 8, 4, 2, 3, 5, 7, in float64:
// the transform is a small part of the path's time, and float64 keeps its
// rounding far below the scores' own float32 noise. Each stage reads every
// butterfly's inputs into registers, synchronises, then writes the outputs in
// place, so one N-point buffer suffices. Rows up to L = 16384 fit one CTA
// (N x 16 bytes <= 128 KB); longer rows are split over a 2-CTA cluster whose
// halves are addressed through distributed shared memory. The N+1 one-sided
// bins come from the even/odd split F_k = E_k + W_L^k O_k; the energy prefix
// and the k* search are float64 warp scans; the low-passed spectrum is
// re-packed the same way and sent through the inverse FFT. Twiddles W_L^m are
// products of two small float64 tables (W_L^{128 hi} W_L^{lo}).
// Prior art on the pages uses cuFFT (AudioKV blog §3.2); this is a
// hand-written transform.
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kSssThreads = 512;
constexpr int kSssWarps = kSssThreads / 32;
constexpr int kMaxPerThread = 16;  // complex values per thread per stage: 8192 / 512
constexpr int kMaxLocal = 8192;    // complex points per CTA (128 KB of float64 pairs)

__device__ __forceinline__ double2 cmul(double2 a, double2 b) {
  return make_double2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ double2 cadd(double2 a, double2 b) { return make_double2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ double2 csub(double2 a, double2 b) { return make_double2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ double2 cconj(double2 a) { return make_double2(a.x, -a.y); }
__device__ __forceinline__ double2 cscale(double2 a, double s) { return make_double2(a.x * s, a.y * s); }
// multiply by -i (forward) or +i (inverse)
__device__ __forceinline__ double2 rot(double2 a, bool inv) {
  return inv ? make_double2(-a.y, a.x) : make_double2(a.y, -a.x);
}

// W_L^m = exp(-2 pi i m / L), 0 <= m < L.
struct Twiddles {
  const double2* lo;  // [128]  W^lo
  const double2* hi;  // [L/128 + 1]  W^{128 hi}
  __device__ __forceinline__ double2 w(int m) const { return cmul(hi[m >> 7], lo[m & 127]); }
};

// The row's N points, split over the cluster's CTAs: [0, half) in rank 0,
// [half, N) in rank 1 (generic pointers reach the other CTA's shared memory).
struct Buf {
  double2* p0;
  double2* p1;
  int half;
  __device__ __forceinline__ double2& at(int m) const { return m < half ? p0[m] : p1[m - half]; }
};

template <int C>
__device__ __forceinline__ void csync(cg::cluster_group& cl) {
  if (C > 1) cl.sync();
  else __syncthreads();
}

template <int RAD>
__device__ __forceinline__ void small_dft(double2 (&v)[RAD], bool inv);

template <>
__device__ __forceinline__ void small_dft<2>(double2 (&v)[2], bool) {
  const double2 a = v[0], b = v[1];
  v[0] = cadd(a, b);
  v[1] = csub(a, b);
}

template <>
__device__ __forceinline__ void small_dft<4>(double2 (&v)[4], bool inv) {
  const double2 a0 = cadd(v[0], v[2]), a1 = csub(v[0], v[2]);
  const double2 a2 = cadd(v[1], v[3]), a3 = rot(csub(v[1], v[3]), inv);
  v[0] = cadd(a0, a2);
  v[2] = csub(a0, a2);
  v[1] = cadd(a1, a3);
  v[3] = csub(a1, a3);
}

template <>
__device__ __forceinline__ void small_dft<8>(double2 (&v)[8], bool inv) {
  double2 e[4] = {v[0], v[2], v[4], v[6]};
  double2 o[4] = {v[1], v[3], v[5], v[7]};
  small_dft<4>(e, inv);
  small_dft<4>(o, inv);
  const double h = 0.70710678118654752440;  // 1/sqrt(2)
  // W8^k O_k with W8 = exp(-+ i pi / 4)
  const double2 o1 = inv ? make_double2(h * (o[1].x - o[1].y), h * (o[1].x + o[1].y))
                         : make_double2(h * (o[1].x + o[1].y), h * (o[1].y - o[1].x));
  const double2 o2 = rot(o[2], inv);
  const double2 o3 = inv ? make_double2(-h * (o[3].x + o[3].y), h * (o[3].x - o[3].y))
                         : make_double2(h * (o[3].y - o[3].x), -h * (o[3].x + o[3].y));
  v[0] = cadd(e[0], o[0]);
  v[4] = csub(e[0], o[0]);
  v[1] = cadd(e[1], o1);
  v[5] = csub(e[1], o1);
  v[2] = cadd(e[2], o2);
  v[6] = csub(e[2], o2);
  v[3] = cadd(e[3], o3);
  v[7] = csub(e[3], o3);
}

// Odd radices by the definition X_k = sum_r v_r W_R^{rk}.
template <int RAD>
__device__ __forceinline__ void odd_dft(double2 (&v)[RAD], bool inv, const double (&cs)[RAD],
                                        const double (&sn)[RAD]) {
  double2 out[RAD];
#pragma unroll
  for (int k = 0; k < RAD; ++k) {
    double2 acc = v[0];
#pragma unroll
    for (int r = 1; r < RAD; ++r) {
      const int m = (r * k) % RAD;
      acc = cadd(acc, cmul(v[r], make_double2(cs[m], inv ? sn[m] : -sn[m])));
    }
    out[k] = acc;
  }
#pragma unroll
  for (int k = 0; k < RAD; ++k) v[k] = out[k];
}

// cos / sin (2 pi m / R): the exact mathematical constants, to double precision.
template <>
__device__ __forceinline__ void small_dft<3>(double2 (&v)[3], bool inv) {
  const double cs[3] = {1.0, -0.5, -0.5};
  const double sn[3] = {0.0, 0.86602540378443864676, -0.86602540378443864676};
  odd_dft<3>(v, inv, cs, sn);
}
template <>
__device__ __forceinline__ void small_dft<5>(double2 (&v)[5], bool inv) {
  const double cs[5] = {1.0, 0.30901699437494742410, -0.80901699437494742410, -0.80901699437494742410,
                        0.30901699437494742410};
  const double sn[5] = {0.0, 0.95105651629515357212, 0.58778525229247312917, -0.58778525229247312917,
                        -0.95105651629515357212};
  odd_dft<5>(v, inv, cs, sn);
}
template <>
__device__ __forceinline__ void small_dft<7>(double2 (&v)[7], bool inv) {
  const double cs[7] = {1.0,
                        0.62348980185873353053,
                        -0.22252093395631440429,
                        -0.90096886790241912624,
                        -0.90096886790241912624,
                        -0.22252093395631440429,
                        0.62348980185873353053};
  const double sn[7] = {0.0,
                        0.78183148246802980871,
                        0.97492791218182360702,
                        0.43388373911755812048,
                        -0.43388373911755812048,
                        -0.97492791218182360702,
                        -0.78183148246802980871};
  odd_dft<7>(v, inv, cs, sn);
}

// One Stockham stage: butterflies j < N / RAD read x[j + r N / RAD], apply
// the twiddles W_{Ns RAD}^{(j mod Ns) r}, transform, and write to
// (j / Ns) Ns RAD + (j mod Ns) + r Ns. The CTAs of a cluster split the
// butterflies into contiguous ranges.
template <int RAD, int C>
__device__ __noinline__ void fft_stage(const Buf& buf, int N, int Ns, int L, bool inv, const Twiddles& tw,
                                       int rank, cg::cluster_group& cl) {
  // a CTA holds at most kMaxLocal points: nb / C <= kMaxLocal / RAD butterflies, at
  // most ceil(kMaxPerThread / RAD) per thread (every one held across the barrier)
  constexpr int MAXB = (kMaxPerThread + RAD - 1) / RAD;
  const int nb = N / RAD;
  const int jb0 = (int)((long long)nb * rank / C), jb1 = (int)((long long)nb * (rank + 1) / C);
  double2 v[MAXB][RAD];
#pragma unroll
  for (int b = 0; b < MAXB; ++b) {
    const int j = jb0 + threadIdx.x + b * kSssThreads;
    if (j < jb1) {
#pragma unroll
      for (int r = 0; r < RAD; ++r) v[b][r] = buf.at(j + r * nb);
    }
  }
  csync<C>(cl);
  const int step = L / (Ns * RAD);  // W_{Ns RAD} = W_L^{step}
#pragma unroll
  for (int b = 0; b < MAXB; ++b) {
    const int j = jb0 + threadIdx.x + b * kSssThreads;
    if (j < jb1) {
      const int k = j % Ns;
#pragma unroll
      for (int r = 1; r < RAD; ++r) {
        double2 w = tw.w(k * r * step);
        if (inv) w.y = -w.y;
        v[b][r] = cmul(v[b][r], w);
      }
      small_dft<RAD>(v[b], inv);
      const int idxD = (j / Ns) * Ns * RAD + k;
#pragma unroll
      for (int r = 0; r < RAD; ++r) buf.at(idxD + r * Ns) = v[b][r];
    }
  }
  csync<C>(cl);
}

template <int C>
__device__ void fft(const Buf& buf, int N, int L, bool inv, const Twiddles& tw, int rank, cg::cluster_group& cl) {
  int rest = N, Ns = 1;
  while (rest > 1) {
    int rad;
    if (rest % 8 == 0) rad = 8;
    else if (rest % 4 == 0) rad = 4;
    else if (rest % 2 == 0) rad = 2;
    else if (rest % 3 == 0) rad = 3;
    else if (rest % 5 == 0) rad = 5;
    else rad = 7;  // lengths with other prime factors are rejected on the host
    switch (rad) {
      case 8: fft_stage<8, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
      case 4: fft_stage<4, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
      case 2: fft_stage<2, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
      case 3: fft_stage<3, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
      case 5: fft_stage<5, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
      default: fft_stage<7, C>(buf, N, Ns, L, inv, tw, rank, cl); break;
    }
    Ns *= rad;
    rest /= rad;
  }
}

__device__ __forceinline__ double warp_incl_scan(double x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// |F_k|^2 for the packing slot 0 = (F_0, F_N), slot k = F_k.
__device__ __forceinline__ double bin_energy(const Buf& buf, int k, int N) {
  if (k == 0) {
    const double f = buf.at(0).x;
    return f * f;
  }
  if (k == N) {
    const double f = buf.at(0).y;
    return f * f;
  }
  const double2 f = buf.at(k);
  return f.x * f.x + f.y * f.y;
}

template <int C>
__global__ void __launch_bounds__(kSssThreads, 1)
    sss_kernel(const RowMap map, const float* __restrict__ s, float* __restrict__ s_hat,
               int32_t* __restrict__ kstar_out, float alpha, float rho) {
  extern __shared__ double2 zb[];
  __shared__ double2 t_lo[128];
  __shared__ double2 t_hi[KV_MAX_L / 128 + 1];
  __shared__ double wsum[kSssWarps];
  __shared__ double cta_sum;
  __shared__ int kmin;

  cg::cluster_group cl = cg::this_cluster();
  const int rank = C > 1 ? (int)cl.block_rank() : 0;
  const int row = blockIdx.x / C;
  const int L = row_len(map, row);
  const int N = L / 2;
  const long long koff = row_key_off(map, row);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Buf buf;
  buf.half = (N + C - 1) / C;
  buf.p0 = C > 1 ? cl.map_shared_rank(zb, 0) : zb;
  buf.p1 = C > 1 ? cl.map_shared_rank(zb, 1) : zb;
  const int m0 = rank * buf.half, m1 = min(N, m0 + buf.half);  // points this CTA holds

  for (int i = threadIdx.x; i < 128; i += kSssThreads) {
    double sv, cv;
    sincospi(2.0 * i / L, &sv, &cv);
    t_lo[i] = make_double2(cv, -sv);
  }
  for (int i = threadIdx.x; i <= L / 128; i += kSssThreads) {
    double sv, cv;
    sincospi(2.0 * (128.0 * i) / L, &sv, &cv);
    t_hi[i] = make_double2(cv, -sv);
  }
  const float2* srow = reinterpret_cast<const float2*>(s + koff);
  for (int m = m0 + threadIdx.x; m < m1; m += kSssThreads) {
    const float2 x = srow[m];
    zb[m - m0] = make_double2(x.x, x.y);
  }
  if (threadIdx.x == 0) kmin = N;
  csync<C>(cl);
  const Twiddles tw{t_lo, t_hi};

  // forward complex FFT of the packed row
  fft<C>(buf, N, L, false, tw, rank, cl);

  // one-sided bins: slot 0 = (F_0, F_N), slot k = F_k for 0 < k < N; the
  // pairs (k, N - k) are split over the cluster by k
  {
    const int np = N / 2 + 1;
    const int k0 = (int)((long long)np * rank / C), k1 = (int)((long long)np * (rank + 1) / C);
    for (int k = k0 + threadIdx.x; k < k1; k += kSssThreads) {
      if (k == 0) {
        const double2 z0 = buf.at(0);
        buf.at(0) = make_double2(z0.x + z0.y, z0.x - z0.y);
      } else {
        const double2 zk = buf.at(k), zm = buf.at(N - k);
        const double2 E = cscale(cadd(zk, cconj(zm)), 0.5);
        const double2 O = cscale(rot(csub(zk, cconj(zm)), false), 0.5);
        const double2 WO = cmul(tw.w(k), O);
        buf.at(k) = cadd(E, WO);
        if (N - k != k) buf.at(N - k) = cconj(csub(E, WO));
      }
    }
  }
  csync<C>(cl);

  // energy prefix over bins 0..N and k* = first k with E(k) >= rho E(N);
  // each CTA scans the bins it holds (bin N sits with slot 0)
  const int b0c = rank == 0 ? 0 : m0, b1c = rank == C - 1 ? N + 1 : m1;
  const int nb_c = max(0, b1c - b0c);
  const int chunk = ((nb_c + kSssWarps - 1) / kSssWarps + 31) & ~31;
  const int b0 = b0c + warp * chunk, b1 = min(b1c, b0 + chunk);
  double part = 0.0;
  for (int k = b0 + lane; k < b1; k += 32) part += bin_energy(buf, k, N);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) wsum[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < kSssWarps; ++i) t += wsum[i];
    cta_sum = t;
  }
  csync<C>(cl);
  double before = 0.0, total = 0.0;
  for (int r = 0; r < C; ++r) {
    const double t = C > 1 ? *cl.map_shared_rank(&cta_sum, r) : cta_sum;
    if (r < rank) before += t;
    total += t;
  }
  for (int i = 0; i < warp; ++i) before += wsum[i];
  const double thr = (double)rho * total;
  double run = before;
  for (int base = b0; base < b1; base += 32) {
    const int k = base + lane;
    const double e = k < b1 ? bin_energy(buf, k, N) : 0.0;
    const double E = run + warp_incl_scan(e);
    const unsigned hit = __ballot_sync(0xffffffffu, k < b1 && E >= thr);
    if (hit) {
      if (lane == 0) atomicMin(&kmin, base + __ffs(hit) - 1);
      break;
    }
    run = __shfl_sync(0xffffffffu, E, 31);
  }
  csync<C>(cl);
  int ks = kmin;
  if (C > 1)
    for (int r = 0; r < C; ++r) ks = min(ks, *cl.map_shared_rank(&kmin, r));

  // low-pass and re-pack for the inverse: Z'_k = E'_k + i O'_k with
  // E'_k = (G_k + conj G_{N-k}) / 2, O'_k = (G_k - conj G_{N-k}) W_L^{-k} / 2
  {
    const int np = N / 2 + 1;
    const int k0 = (int)((long long)np * rank / C), k1 = (int)((long long)np * (rank + 1) / C);
    for (int k = k0 + threadIdx.x; k < k1; k += kSssThreads) {
      if (k == 0) {
        const double2 z0 = buf.at(0);
        const double g0 = z0.x;
        const double gN = ks >= N ? z0.y : 0.0;
        buf.at(0) = make_double2(0.5 * (g0 + gN), 0.5 * (g0 - gN));
      } else {
        const double2 zero = make_double2(0.0, 0.0);
        const double2 gk = k <= ks ? buf.at(k) : zero;
        const double2 gm = (N - k) <= ks ? buf.at(N - k) : zero;
        const double2 E = cscale(cadd(gk, cconj(gm)), 0.5);
        const double2 O = cmul(cscale(csub(gk, cconj(gm)), 0.5), cconj(tw.w(k)));
        buf.at(k) = make_double2(E.x - O.y, E.y + O.x);  // E + i O
        if (N - k != k) buf.at(N - k) = make_double2(E.x + O.y, -E.y + O.x);  // conj(E) + i conj(O)
      }
    }
  }
  csync<C>(cl);

  fft<C>(buf, N, L, true, tw, rank, cl);

  const double inv_n = 1.0 / (double)N;
  const double a = alpha;
  float2* hrow = reinterpret_cast<float2*>(s_hat + koff);
  for (int m = m0 + threadIdx.x; m < m1; m += kSssThreads) {
    const double2 y = zb[m - m0];
    const float2 x = srow[m];
    hrow[m] = make_float2((float)((1.0 - a) * x.x + a * (y.x * inv_n)), (float)((1.0 - a) * x.y + a * (y.y * inv_n)));
  }
  if (rank == 0 && threadIdx.x == 0) kstar_out[row] = ks;
  if (C > 1) cl.sync();  // no CTA leaves while the other may still read its shared memory
}

}  // namespace

int launch_sss(const RowMap& m, const float* s, float* s_hat, int32_t* kstar, float alpha, float rho,
               cudaStream_t st) {
  int maxN = 0;
  for (int i = 0; i < m.n_seq; ++i) maxN = std::max(maxN, m.L[i] / 2);
  const int C = maxN > kMaxLocal ? 2 : 1;
  const int local = (maxN + C - 1) / C;
  const size_t smem = (size_t)local * sizeof(double2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(m.n_rows * C);
  cfg.blockDim = dim3(kSssThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (C == 1) {
    e = cudaFuncSetAttribute(sss_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, sss_kernel<1>, m, s, s_hat, kstar, alpha, rho);
  } else {
    e = cudaFuncSetAttribute(sss_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, sss_kernel<2>, m, s, s_hat, kstar, alpha, rho);
  }
  return cuda_status(e);
}

}  // namespace kvc
