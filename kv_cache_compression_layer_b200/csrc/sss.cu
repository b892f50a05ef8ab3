// kv_sss: Spectral Score Smoothing (AudioKV blog §2.2).
//
//   F = RFFT(s);  E(k) = sum_{i<=k} |F_i|^2;  k* = min{k : E(k) >= rho E(L/2)};
//   s_hat = (1 - alpha) s + alpha IRFFT(F 1[i <= k*], n = L).
//
// The real row of even length L is packed as N = L/2 complex points
// z_m = s_{2m} + i s_{2m+1} and transformed in place in shared memory, in
// float64 (the transform is a small part of the path's time, and float64 keeps
// its rounding far below the scores' own float32 noise). The forward transform
// is a mixed-radix decimation in frequency (radices 8, 4, 2, 3, 5, 7 in that
// order of preference): each butterfly reads its R points, takes their R-point
// DFT, multiplies by the twiddles and writes the same R points back, so a stage
// is one pass and one barrier with nothing held across it. It leaves Z_k at the
// digit-reversed position rev(k) (k's mixed-radix digits read in reverse
// order), and the spectrum is worked on in place through a table of rev: the
// N+1 one-sided bins come from the even/odd split F_k = E_k + W_L^k O_k, the
// energy prefix and the k* search are float64 warp scans over k in natural
// order, and the low-passed spectrum is re-packed the same way. The inverse is
// the matching decimation in time, stage by stage in reverse, which takes the
// digit-reversed spectrum back to natural order. Odd radices use the
// conjugate-pair form of the DFT (x_n +/- x_{R-n} against cosines and sines).
// Twiddles W_L^m are products of two small float64 tables
// (W_L^{128 hi} W_L^{lo}); a butterfly's k-th twiddle is the k-th power of its
// first.
//
// Rows with N <= 2048 are taken four to a CTA and N <= 4096 two (a named
// barrier per row), N <= 8192 one; longer rows are split over a 2-CTA cluster
// whose halves are addressed through distributed shared memory. A batch that
// would leave SMs idle that way (fewer CTAs than SMs) gets one row per CTA. Sequences are
// launched longest first. Prior art on the pages uses cuFFT (AudioKV blog
// §3.2); this is a hand-written transform.
#include <algorithm>
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kSssThreads = 512;
constexpr int kSssWarps = kSssThreads / 32;
constexpr int kMaxLocal = 8192;  // complex points of one CTA's buffer (128 KB of float64 pairs)
constexpr int kMaxStages = 16;
constexpr int kMaxPer = kMaxLocal / kSssThreads;  // points per thread: a CTA's buffer over its threads
constexpr int kTwHi = KV_MAX_L / 128 + 1;

// Shared-memory layout: twiddle tables, the rev table, the point buffer.
template <int C>
struct SssLayout {
  static constexpr int kRevCap = C * kMaxLocal;  // rev entries (the whole row's N)
  static constexpr size_t kTwBytes = (size_t)(kTwHi + 128) * 16;
  static constexpr size_t kDataOff = (kTwBytes + (size_t)kRevCap * 2 + 15) & ~size_t(15);
  static constexpr size_t kBytes = kDataOff + (size_t)kMaxLocal * 16;
};

// Sequences of one launch: longest first, each with its rows per CTA (cluster)
// and its first CTA (cluster).
struct SssPlan {
  int n;
  int seq[KV_MAX_SEQ];
  int per[KV_MAX_SEQ];
  int first[KV_MAX_SEQ + 1];
};

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

// A row's N points: one CTA's shared memory, or a cluster's two halves
// ([0, half) in rank 0, [half, N) in rank 1; generic pointers reach the other
// CTA's shared memory).
// With SWZ the points of each 128-byte row (8 points) are permuted by an XOR
// of higher index bits: for N a multiple of 64 the spectrum's digit-reversed
// positions of consecutive k lie a multiple of 8 points apart, and would
// otherwise all fall on the same shared-memory banks.
template <bool SWZ>
__device__ __forceinline__ int swz(int m) {
  return SWZ ? m ^ (((m >> 3) ^ (m >> 6) ^ (m >> 9) ^ (m >> 12)) & 7) : m;
}
template <bool SWZ>
struct LocalBuf {
  double2* p;
  __device__ __forceinline__ double2& at(int m) const { return p[swz<SWZ>(m)]; }
};
template <bool SWZ>
struct ClusterBuf {  // half is a multiple of 8: a row never straddles the halves
  double2* p0;
  double2* p1;
  int half;
  __device__ __forceinline__ double2& at(int m) const {
    const int q = swz<SWZ>(m);
    return q < half ? p0[q] : p1[q - half];
  }
};

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

// Odd radices in conjugate pairs: with theta = 2 pi n k / R,
//   X_k, X_{R-k} = x_0 + sum_{n=1}^{(R-1)/2} (x_n + x_{R-n}) cos theta  -/+  i sum (x_n - x_{R-n}) sin theta
// (the signs swap for the inverse).
template <int RAD>
__device__ __forceinline__ void odd_dft(double2 (&v)[RAD], bool inv, const double (&cs)[RAD],
                                        const double (&sn)[RAD]) {
  constexpr int H = (RAD - 1) / 2;
  double2 t[H], d[H];
#pragma unroll
  for (int n = 1; n <= H; ++n) {
    t[n - 1] = cadd(v[n], v[RAD - n]);
    d[n - 1] = csub(v[n], v[RAD - n]);
  }
  const double2 x0 = v[0];
  double2 sum = x0;
#pragma unroll
  for (int n = 0; n < H; ++n) sum = cadd(sum, t[n]);
#pragma unroll
  for (int k = 1; k <= H; ++k) {
    double2 a = x0, b = make_double2(0.0, 0.0);
#pragma unroll
    for (int n = 1; n <= H; ++n) {
      const int m = (n * k) % RAD;
      a = make_double2(fma(t[n - 1].x, cs[m], a.x), fma(t[n - 1].y, cs[m], a.y));
      b = make_double2(fma(d[n - 1].x, sn[m], b.x), fma(d[n - 1].y, sn[m], b.y));
    }
    // -i b = (b.y, -b.x)
    const double2 mib = make_double2(b.y, -b.x);
    v[k] = inv ? csub(a, mib) : cadd(a, mib);
    v[RAD - k] = inv ? cadd(a, mib) : csub(a, mib);
  }
  v[0] = sum;
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

// One stage on blocks of B = RAD S points: butterfly t (block t / S, offset
// n' = t mod S) owns the points base + r S, base = (t / S) B + n'.
//   forward (decimation in frequency): DFT over r, then point k times W_B^{n' k};
//   inverse (decimation in time): point k times W_B^{-n' k}, then the inverse DFT.
// Butterflies [t0, t1) are taken by this thread with stride `step`.
template <int RAD, bool INV, class Buf>
__device__ __forceinline__ void butterfly(const Buf& z, int t, int S, unsigned magic, int lstep, const Twiddles& tw,
                                          double2 (&v)[RAD], int& base, int& np) {
  const int blk = S == 1 ? t : (int)__umulhi((unsigned)t, magic);  // t / S (exact for t S < 2^32)
  np = t - blk * S;
  base = blk * RAD * S + np;
#pragma unroll
  for (int r = 0; r < RAD; ++r) v[r] = z.at(base + r * S);
}
template <int RAD, bool INV>
__device__ __forceinline__ void butterfly_math(double2 (&v)[RAD], int np, int lstep, const Twiddles& tw) {
  if (!INV) small_dft<RAD>(v, false);
  if (np != 0) {
    double2 w1 = tw.w(np * lstep);
    if (INV) w1 = cconj(w1);
    double2 w = w1;
#pragma unroll
    for (int k = 1; k < RAD; ++k) {
      v[k] = cmul(v[k], w);
      if (k + 1 < RAD) w = cmul(w, w1);
    }
  }
  if (INV) small_dft<RAD>(v, true);
}

// One stage on blocks of B = RAD S points: butterfly t (block t / S, offset
// n' = t mod S) owns the points base + r S, base = (t / S) B + n'.
//   forward (decimation in frequency): DFT over r, then point k times W_B^{n' k};
//   inverse (decimation in time): point k times W_B^{-n' k}, then the inverse DFT.
// Butterflies [t0, t1) are taken by this thread with stride `step`; up to
// radix 5 two at a time (their points are disjoint: both are read before
// either is written).
template <int RAD, bool INV, class Buf>
__device__ __forceinline__ void fft_stage(const Buf& z, int S, int L, const Twiddles& tw, int t0, int t1,
                                          int step) {
  const int lstep = L / (RAD * S);  // W_B = W_L^{lstep}
  const unsigned magic = S == 1 ? 0u : (unsigned)((0x100000000ull + (unsigned)S - 1) / (unsigned)S);
  int t = t0;
  for (; RAD <= 5 && t + step < t1; t += 2 * step) {
    double2 v[RAD], u[RAD];
    int bv, nv, bu, nu;
    butterfly<RAD, INV>(z, t, S, magic, lstep, tw, v, bv, nv);
    butterfly<RAD, INV>(z, t + step, S, magic, lstep, tw, u, bu, nu);
    butterfly_math<RAD, INV>(v, nv, lstep, tw);
    butterfly_math<RAD, INV>(u, nu, lstep, tw);
#pragma unroll
    for (int k = 0; k < RAD; ++k) z.at(bv + k * S) = v[k];
#pragma unroll
    for (int k = 0; k < RAD; ++k) z.at(bu + k * S) = u[k];
  }
  for (; t < t1; t += step) {
    double2 v[RAD];
    int bv, nv;
    butterfly<RAD, INV>(z, t, S, magic, lstep, tw, v, bv, nv);
    butterfly_math<RAD, INV>(v, nv, lstep, tw);
#pragma unroll
    for (int k = 0; k < RAD; ++k) z.at(bv + k * S) = v[k];
  }
}

// The whole transform: forward stages in plan order (block B from N down), or
// the inverse stages in reverse order (span S from 1 up). `sync` is the row's barrier.
template <bool INV, class Buf, class Sync>
__device__ __forceinline__ void fft(const Buf& z, int N, int L, const int* rad, int m, const Twiddles& tw,
                                    int bnum, int bden, int tid, int step, Sync sync) {
  int S = INV ? 1 : N;
  for (int i = 0; i < m; ++i) {
    const int s = INV ? m - 1 - i : i;
    const int R = rad[s];
    if (!INV) S /= R;
    const int nb = N / R;
    // this CTA's butterflies (a cluster's CTAs take contiguous shares), then this thread's
    const int c0 = (int)((long long)nb * bnum / bden);
    const int c1 = (int)((long long)nb * (bnum + 1) / bden);
    switch (R) {
      case 8: fft_stage<8, INV>(z, S, L, tw, c0 + tid, c1, step); break;
      case 4: fft_stage<4, INV>(z, S, L, tw, c0 + tid, c1, step); break;
      case 2: fft_stage<2, INV>(z, S, L, tw, c0 + tid, c1, step); break;
      case 3: fft_stage<3, INV>(z, S, L, tw, c0 + tid, c1, step); break;
      case 5: fft_stage<5, INV>(z, S, L, tw, c0 + tid, c1, step); break;
      default: fft_stage<7, INV>(z, S, L, tw, c0 + tid, c1, step); break;
    }
    sync();
    if (INV) S *= R;
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

template <int C>
__global__ void __launch_bounds__(kSssThreads, 1)
    sss_kernel(const RowMap map, const SssPlan plan, const float* __restrict__ s, float* __restrict__ s_hat,
               int32_t* __restrict__ kstar_out, float alpha, float rho) {
  using Lay = SssLayout<C>;
  extern __shared__ __align__(16) uint8_t sss_smem[];
  double2* t_hi = reinterpret_cast<double2*>(sss_smem);
  double2* t_lo = t_hi + kTwHi;
  uint16_t* rev = reinterpret_cast<uint16_t*>(sss_smem + Lay::kTwBytes);
  double2* zb = reinterpret_cast<double2*>(sss_smem + Lay::kDataOff);
  __shared__ int rad_s[kMaxStages];
  __shared__ unsigned mg_s[kMaxStages];  // per stage: ceil(2^32 / radix), for k / radix by a multiply-high
  __shared__ int blk_s[kMaxStages];      // per stage: N over the product of the radices up to it
  __shared__ int m_s;
  __shared__ double wsum[kSssWarps];
  __shared__ double gsum[4];
  __shared__ int kmin_s[4];

  cg::cluster_group cl = cg::this_cluster();
  const int rank = C > 1 ? (int)cl.block_rank() : 0;
  const int unit = blockIdx.x / C;  // CTA (cluster) of the launch
  int q = 0;
  while (q + 1 < plan.n && plan.first[q + 1] <= unit) ++q;
  const int seq = plan.seq[q], P = plan.per[q];
  const int L = map.L[seq], N = L / 2;
  const int T = kSssThreads / P;  // threads per row
  const int g = threadIdx.x / T, tg = threadIdx.x - g * T;
  const int row_in_seq = (unit - plan.first[q]) * P + g;
  const bool live = row_in_seq < map.rows_per_seq;
  const int row = seq * map.rows_per_seq + row_in_seq;
  const int lane = threadIdx.x & 31;

  // shared tables of the CTA (every row of it has this L)
  if (threadIdx.x == 0) {
    int rest = N, m = 0;
    while (rest > 1) {
      int r;
      if (rest % 8 == 0) r = 8;
      else if (rest % 4 == 0) r = 4;
      else if (rest % 2 == 0) r = 2;
      else if (rest % 3 == 0) r = 3;
      else if (rest % 5 == 0) r = 5;
      else r = 7;  // lengths with other prime factors are rejected on the host
      rad_s[m] = r;
      mg_s[m] = (unsigned)((0x100000000ull + (unsigned)r - 1) / (unsigned)r);
      rest /= r;
      blk_s[m++] = rest;
    }
    m_s = m;
  }
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
  if (threadIdx.x < 4) kmin_s[threadIdx.x] = N;
  const int half = (N + C - 1) / C;
  const int m0 = rank * half, m1 = min(N, m0 + half);  // points this CTA holds (C = 2)
  const int pm0 = C > 1 ? m0 : 0, pm1 = C > 1 ? m1 : N;  // this CTA's points of the row
  const long long koff = live ? row_key_off(map, row) : 0;
  const float2* srow = reinterpret_cast<const float2*>(s + koff);
  __syncthreads();
  const int m = m_s;
  // rev(k): k's digits (first radix lowest) reversed, stage by stage over this
  // thread's indices k = threadIdx.x + j 512
  constexpr int kRevPer = 8;
  for (int k0 = 0; k0 < N; k0 += kRevPer * kSssThreads) {
    int kk[kRevPer], pos[kRevPer];
#pragma unroll
    for (int j = 0; j < kRevPer; ++j) {
      kk[j] = k0 + (int)threadIdx.x + j * kSssThreads;
      pos[j] = 0;
    }
    for (int i = 0; i < m; ++i) {
      const int r = rad_s[i], B = blk_s[i];
      const unsigned mg = mg_s[i];  // kk / r for kk < 2^16
#pragma unroll
      for (int j = 0; j < kRevPer; ++j) {
        const int q = (int)__umulhi((unsigned)kk[j], mg);
        pos[j] += (kk[j] - q * r) * B;
        kk[j] = q;
      }
    }
#pragma unroll
    for (int j = 0; j < kRevPer; ++j) {
      const int k = k0 + (int)threadIdx.x + j * kSssThreads;
      if (k < N) rev[k] = (uint16_t)pos[j];
    }
  }
  if (C > 1) cl.sync();  // both halves exist and the tables are in place
  else __syncthreads();
  if (!live) return;  // no CTA-wide barrier follows

  const Twiddles tw{t_lo, t_hi};
  auto sync = [&]() {
    if (C > 1) cl.sync();
    else if (P == 1) __syncthreads();
    else named_bar_sync(1 + g, T);
  };
  float2* hrow = reinterpret_cast<float2*>(s_hat + koff);
  const bool sw = N % 64 == 0;  // the spectrum's digit-reversed accesses would hit the same banks

  // the row's points; the transform, the spectrum and the blend
  // z0 addresses the points plainly (the transforms); z through the row swizzle when
  // sw (the spectrum work); permute moves this CTA's points between the two layouts
  // (the swizzle is its own inverse and stays inside 8-point rows, so inside a half)
  auto run = [&](const auto& z0, const auto& z, int tid, int step, int bnum, int bden) {
    // for each j the threads' points pm0 + tid + j step are whole 8-point rows, so the
    // permutation is done eight j at a time
    auto permute = [&](const auto& zz) {
#pragma unroll
      for (int j0 = 0; j0 < kMaxPer; j0 += 8) {
        double2 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = pm0 + tid + (j0 + j) * step;
          if (i < pm1) v[j] = zz.at(i);
        }
        sync();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = pm0 + tid + (j0 + j) * step;
          if (i < pm1) zz.at(swz<true>(i)) = v[j];
        }
        sync();
      }
    };
#pragma unroll 1
    for (int j0 = 0; j0 < kMaxPer; j0 += 8) {  // eight of the thread's points' loads in flight at a time
      float2 x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = pm0 + tid + (j0 + j) * step;
        if (i < pm1) x[j] = srow[i];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = pm0 + tid + (j0 + j) * step;
        if (i < pm1) z0.at(i) = make_double2(x[j].x, x[j].y);
      }
    }
    sync();
    fft<false>(z0, N, L, rad_s, m, tw, bnum, bden, tid, step, sync);
    if (sw) permute(z0);

    // one-sided bins: slot rev(0) = 0 holds (F_0, F_N), slot rev(k) holds F_k; the
    // pairs (k, N - k) are split over the cluster by k
    const int np = N / 2 + 1;
    const int k0 = (int)((long long)np * bnum / bden), k1 = (int)((long long)np * (bnum + 1) / bden);
    for (int k = k0 + tid; k < k1; k += step) {
      if (k == 0) {
        const double2 z0 = z.at(0);
        z.at(0) = make_double2(z0.x + z0.y, z0.x - z0.y);
      } else {
        const int pk = rev[k], pm = rev[N - k];
        const double2 zk = z.at(pk), zm = z.at(pm);
        const double2 E = cscale(cadd(zk, cconj(zm)), 0.5);
        const double2 O = cscale(rot(csub(zk, cconj(zm)), false), 0.5);
        const double2 WO = cmul(tw.w(k), O);
        z.at(pk) = cadd(E, WO);
        if (N - k != k) z.at(pm) = cconj(csub(E, WO));
      }
    }
    sync();

    // energy prefix over bins 0..N in natural order and k* = first k with
    // E(k) >= rho E(N); a cluster's CTAs scan contiguous halves of the bins
    auto bin_energy = [&](int k) -> double {
      if (k == 0) {
        const double f = z.at(0).x;
        return f * f;
      }
      if (k == N) {
        const double f = z.at(0).y;
        return f * f;
      }
      const double2 f = z.at(rev[k]);
      return f.x * f.x + f.y * f.y;
    };
    const int nbins = N + 1;
    const int kb0 = (int)((long long)nbins * bnum / bden), kb1 = (int)((long long)nbins * (bnum + 1) / bden);
    const int nw = step / 32, gw = tid >> 5, wbase = (threadIdx.x >> 5) - gw;  // the row's warps
    const int chunk = ((kb1 - kb0 + nw - 1) / nw + 31) & ~31;
    const int b0 = kb0 + gw * chunk, b1 = min(kb1, b0 + chunk);
    double part = 0.0;
    for (int k = b0 + lane; k < b1; k += 32) part += bin_energy(k);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) wsum[wbase + gw] = part;
    sync();
    if (tid == 0) {
      double t = 0.0;
      for (int i = 0; i < nw; ++i) t += wsum[wbase + i];
      gsum[g] = t;
    }
    sync();
    double before = 0.0, total = 0.0;
    if (C > 1) {
      for (int r = 0; r < C; ++r) {
        const double t = *cl.map_shared_rank(&gsum[0], r);
        if (r < rank) before += t;
        total += t;
      }
    } else {
      total = gsum[g];
    }
    for (int i = 0; i < gw; ++i) before += wsum[wbase + i];
    const double thr = (double)rho * total;
    double run_e = before;
    for (int base = b0; base < b1; base += 32) {
      const int k = base + lane;
      const double e = k < b1 ? bin_energy(k) : 0.0;
      const double Ek = run_e + warp_incl_scan(e);
      const unsigned hit = __ballot_sync(0xffffffffu, k < b1 && Ek >= thr);
      if (hit) {
        if (lane == 0) atomicMin(&kmin_s[g], base + __ffs(hit) - 1);
        break;
      }
      run_e = __shfl_sync(0xffffffffu, Ek, 31);
    }
    sync();
    int ks = kmin_s[g];
    if (C > 1)
      for (int r = 0; r < C; ++r) ks = min(ks, *cl.map_shared_rank(&kmin_s[0], r));

    // low-pass and re-pack for the inverse: Z'_k = E'_k + i O'_k with
    // E'_k = (G_k + conj G_{N-k}) / 2, O'_k = (G_k - conj G_{N-k}) W_L^{-k} / 2
    for (int k = k0 + tid; k < k1; k += step) {
      if (k == 0) {
        const double2 z0 = z.at(0);
        const double g0 = z0.x;
        const double gN = ks >= N ? z0.y : 0.0;
        z.at(0) = make_double2(0.5 * (g0 + gN), 0.5 * (g0 - gN));
      } else {
        const int pk = rev[k], pm = rev[N - k];
        const double2 zero = make_double2(0.0, 0.0);
        const double2 gk = k <= ks ? z.at(pk) : zero;
        const double2 gm = (N - k) <= ks ? z.at(pm) : zero;
        const double2 E = cscale(cadd(gk, cconj(gm)), 0.5);
        const double2 O = cmul(cscale(csub(gk, cconj(gm)), 0.5), cconj(tw.w(k)));
        z.at(pk) = make_double2(E.x - O.y, E.y + O.x);  // E + i O
        if (N - k != k) z.at(pm) = make_double2(E.x + O.y, -E.y + O.x);  // conj(E) + i conj(O)
      }
    }
    sync();

    if (sw) permute(z0);
    fft<true>(z0, N, L, rad_s, m, tw, bnum, bden, tid, step, sync);

    const double inv_n = 1.0 / (double)N;
    const double a = alpha;
    for (int i = pm0 + tid; i < pm1; i += step) {
      const double2 y = z0.at(i);
      const float2 x = srow[i];
      hrow[i] = make_float2((float)((1.0 - a) * x.x + a * (y.x * inv_n)), (float)((1.0 - a) * x.y + a * (y.y * inv_n)));
    }
    if (bnum == 0 && tid == 0) kstar_out[row] = ks;
  };

  if (C > 1) {
    double2* p0 = cl.map_shared_rank(zb, 0);
    double2* p1 = cl.map_shared_rank(zb, 1);
    const ClusterBuf<false> zp{p0, p1, half};
    if (sw) run(zp, ClusterBuf<true>{p0, p1, half}, (int)threadIdx.x, kSssThreads, rank, C);
    else run(zp, zp, (int)threadIdx.x, kSssThreads, rank, C);
    cl.sync();  // no CTA leaves while the other may still read its shared memory
  } else {
    double2* own = zb + g * N;
    if (sw) run(LocalBuf<false>{own}, LocalBuf<true>{own}, tg, T, 0, 1);
    else run(LocalBuf<false>{own}, LocalBuf<false>{own}, tg, T, 0, 1);
  }
}

}  // namespace

int launch_sss(const RowMap& m, const float* s, float* s_hat, int32_t* kstar, float alpha, float rho,
               cudaStream_t st) {
  // sequences longest first; rows per CTA by length (one when the batch is too
  // small to fill the SMs otherwise); rows past kMaxLocal points on a cluster
  int order[KV_MAX_SEQ];
  for (int i = 0; i < m.n_seq; ++i) order[i] = i;
  std::stable_sort(order, order + m.n_seq, [&](int x, int y) { return m.L[x] > m.L[y]; });
  SssPlan p1 = {}, p2 = {};
  int ctas = 0;
  for (int i = 0; i < m.n_seq; ++i) {
    const int N = m.L[i] / 2;
    const int per = N > kMaxLocal ? 1 : N > 4096 ? 1 : N > 2048 ? 2 : 4;
    ctas += (N > kMaxLocal ? 2 : 1) * ((m.rows_per_seq + per - 1) / per);
  }
  const bool few = ctas < sm_count();
  for (int i = 0; i < m.n_seq; ++i) {
    const int sq = order[i], N = m.L[sq] / 2;
    SssPlan& p = N > kMaxLocal ? p2 : p1;
    const int per = few || N > 4096 ? 1 : N > 2048 ? 2 : 4;
    p.seq[p.n] = sq;
    p.per[p.n] = N > kMaxLocal ? 1 : per;
    p.first[p.n + 1] = p.first[p.n] + (m.rows_per_seq + p.per[p.n] - 1) / p.per[p.n];
    ++p.n;
  }
  cudaError_t e = cudaSuccess;
  if (p1.n > 0) {
    const size_t smem = SssLayout<1>::kBytes;
    e = cudaFuncSetAttribute(sss_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) sss_kernel<1><<<p1.first[p1.n], kSssThreads, smem, st>>>(m, p1, s, s_hat, kstar, alpha, rho);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e == cudaSuccess && p2.n > 0) {
    const size_t smem = SssLayout<2>::kBytes;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * p2.first[p2.n]);
    cfg.blockDim = dim3(kSssThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaFuncSetAttribute(sss_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, sss_kernel<2>, m, p2, s, s_hat, kstar, alpha, rho);
  }
  return cuda_status(e);
}

}  // namespace kvc
