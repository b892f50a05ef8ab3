// kv_c3_build / kv_c3_step: C3's key-space retrieval ("C3: Speech-Guided KV
// Retrieval for Long-Context SpeechLLM Inference"): a bisecting 2-means
// index per (layer, KV head) row, shared-GQA competition of the frontier
// clusters for a budget of B audio keys, exact attention over them, and
// adaptive resolution by a relevance EMA with split/merge exchanges.
//
// The index and the scores are float64 in a fixed operation order (products
// and sums rounded separately, sums in index order), so the tree, the
// frontier and every selection are reproducible bit for bit.
//
// build: per tree level a plan kernel (one CTA per row) numbers the children
// of the level's splitting nodes breadth-first and queues them; a split
// kernel (one CTA per node) runs the 2-means and partitions the node's
// members stably; then a centroid kernel (a warp per node) and a frontier
// kernel (one CTA per row).
// step: a score kernel (a thread per frontier node), a select kernel (one CTA
// per row: a weighted radix select of the cluster where the budget runs out,
// then an ordered compaction of the retrieved positions), an attention kernel
// (one CTA per row and query head) and an update kernel (one CTA per row:
// EMA, exchanges by block argmax/argmin, frontier compaction).
#include <algorithm>
#include <cmath>
#include <cstring>

#include "../../include/kvcomp_next.h"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kHdr = 4;  // int32 words of a row's header: nodes, A, retrieved keys, 0

struct C3Arr {
  uint8_t* base;
  kv_c3_layout lay;
  __host__ __device__ int32_t* perm() const { return reinterpret_cast<int32_t*>(base + lay.perm); }
  __host__ __device__ int32_t* lo() const { return reinterpret_cast<int32_t*>(base + lay.lo); }
  __host__ __device__ int32_t* cnt() const { return reinterpret_cast<int32_t*>(base + lay.cnt); }
  __host__ __device__ int32_t* left() const { return reinterpret_cast<int32_t*>(base + lay.left); }
  __host__ __device__ int32_t* depth() const { return reinterpret_cast<int32_t*>(base + lay.depth); }
  __host__ __device__ double* e() const { return reinterpret_cast<double*>(base + lay.e); }
  __host__ __device__ double* cent() const { return reinterpret_cast<double*>(base + lay.cent); }
  __host__ __device__ int32_t* front() const { return reinterpret_cast<int32_t*>(base + lay.front); }
  __host__ __device__ double* sigma() const { return reinterpret_cast<double*>(base + lay.sigma); }
  __host__ __device__ int32_t* sel() const { return reinterpret_cast<int32_t*>(base + lay.sel); }
  __host__ __device__ int32_t* hdr() const { return reinterpret_cast<int32_t*>(base + lay.hdr); }
  // scratch
  uint8_t* side;   // per key
  int32_t* tmp;    // per key
  uint8_t* taken;  // per key
  uint8_t* on;     // per node
  uint8_t* fresh;  // per node
  int32_t* tasks;  // (row, node) pairs: the splits of the current level
  int32_t* count;  // [4]
  int32_t* parent; // per node: the node it was split from (-1 for the root)
};

// Scratch of the index that the public layout does not name.
struct C3Scratch {
  uint64_t side, tmp, taken, on, fresh, tasks, count, parent;
};

uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

void layout_of(long long T, int rows, int d, kv_c3_layout& L, C3Scratch& S) {
  uint64_t o = 0;
  auto take = [&](uint64_t bytes) {
    const uint64_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  const uint64_t nodes = 2ull * (uint64_t)T;
  L.cent = take(nodes * (uint64_t)d * 8);
  L.e = take(nodes * 8);
  L.sigma = take(nodes * 8);
  L.perm = take((uint64_t)T * 4);
  L.lo = take(nodes * 4);
  L.cnt = take(nodes * 4);
  L.left = take(nodes * 4);
  L.depth = take(nodes * 4);
  L.front = take(nodes * 4);
  L.sel = take((uint64_t)T * 4);
  L.hdr = take((uint64_t)rows * kHdr * 4);
  S.tmp = take((uint64_t)T * 4);
  S.tasks = take((uint64_t)T * 2 * 4);
  S.side = take((uint64_t)T);
  S.taken = take((uint64_t)T);
  S.on = take(nodes);
  S.fresh = take(nodes);
  S.count = take(16);
  S.parent = take(nodes * 4);
  L.bytes = o;
}

C3Arr arrays_of(void* index, const kv_c3_layout& L, const C3Scratch& S) {
  C3Arr a;
  a.base = static_cast<uint8_t*>(index);
  a.lay = L;
  a.side = a.base + S.side;
  a.tmp = reinterpret_cast<int32_t*>(a.base + S.tmp);
  a.taken = a.base + S.taken;
  a.on = a.base + S.on;
  a.fresh = a.base + S.fresh;
  a.tasks = reinterpret_cast<int32_t*>(a.base + S.tasks);
  a.count = reinterpret_cast<int32_t*>(a.base + S.count);
  a.parent = reinterpret_cast<int32_t*>(a.base + S.parent);
  return a;
}

__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9e3779b97f4a7c15ull;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

template <typename T>
__device__ __forceinline__ double ld(const T* p);
template <>
__device__ __forceinline__ double ld<float>(const float* p) {
  return (double)__ldg(p);
}
template <>
__device__ __forceinline__ double ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return (double)__bfloat162float(__ldg(p));
}

constexpr int kScanThreads = 1024;
constexpr int kC3SelReg = 4;  // frontier entries a select thread keeps in registers

// Exclusive sum over a block of kScanThreads threads; *total = the block's sum.
__device__ int scan_excl(int v, int* total, int* sh) {
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
    int w = sh[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh[32 + lane] = w;
  }
  __syncthreads();
  const int before = (warp ? sh[32 + warp - 1] : 0) + x - v;
  *total = sh[63];
  __syncthreads();
  return before;
}

// ------------------------------------------------------------------ build --
__global__ void __launch_bounds__(256) c3_init_kernel(const RowMap m, C3Arr a) {
  const int row = blockIdx.x;
  const int L = row_len(m, row);
  const long long ko = row_key_off(m, row);
  for (int j = threadIdx.x; j < L; j += blockDim.x) a.perm()[ko + j] = j;
  if (threadIdx.x == 0) {
    const long long no = 2 * ko;
    a.lo()[no] = 0;
    a.cnt()[no] = L;
    a.left()[no] = -1;
    a.depth()[no] = 0;
    a.parent[no] = -1;
    int32_t* h = a.hdr() + (long long)row * kHdr;
    h[0] = 1;  // nodes
    h[1] = 0;  // level begin (until the frontier kernel stores A here)
    h[2] = 1;  // level end
    h[3] = 0;
  }
}

// Numbers the children of this level's splitting nodes breadth-first and
// queues the splits as (row, node) pairs.
__global__ void __launch_bounds__(kScanThreads) c3_plan_kernel(const RowMap m, C3Arr a, int leaf_max) {
  __shared__ int sh[64];
  const int row = blockIdx.x;
  const long long no = 2 * row_key_off(m, row);
  int32_t* h = a.hdr() + (long long)row * kHdr;
  const int lb = h[1], le = h[2];
  int carry = 0;
  for (int base = lb; base < le; base += kScanThreads) {
    const int n = base + threadIdx.x;
    const bool split = n < le && a.cnt()[no + n] > leaf_max && a.cnt()[no + n] >= 2;
    int tot;
    const int r = carry + scan_excl(split ? 1 : 0, &tot, sh);
    if (n < le) {
      if (split) {
        const int c = le + 2 * r;
        a.left()[no + n] = c;
        a.depth()[no + c] = a.depth()[no + c + 1] = a.depth()[no + n] + 1;
        a.left()[no + c] = a.left()[no + c + 1] = -1;
        a.parent[no + c] = a.parent[no + c + 1] = n;
        const int q = atomicAdd(a.count, 1);
        a.tasks[2 * q] = row;
        a.tasks[2 * q + 1] = n;
      } else {
        a.left()[no + n] = -1;
      }
    }
    carry += tot;
  }
  if (threadIdx.x == 0) {
    h[0] = le + 2 * carry;
    h[1] = le;
    h[2] = le + 2 * carry;
  }
}

constexpr int kSplitThreads = 256;

// 2-means of one node (the oracle's order: distances summed over the
// dimensions, centroid sums over the members in index order), then a stable
// partition of its members: left side first.
template <typename T>
__global__ void __launch_bounds__(kSplitThreads)
    c3_split_kernel(const RowMap m, C3Arr a, const T* __restrict__ K, int d, int iters, uint64_t seed) {
  __shared__ double c[2][128];
  __shared__ int sh[64];
  __shared__ int n0_s;
  const int row = a.tasks[2 * blockIdx.x], nd = a.tasks[2 * blockIdx.x + 1];
  const long long ko = row_key_off(m, row), no = 2 * ko;
  const int lo = a.lo()[no + nd], n = a.cnt()[no + nd];
  int32_t* mem = a.perm() + ko + lo;
  uint8_t* side = a.side + ko + lo;
  const T* Kr = K + ko * d;
  const int tid = threadIdx.x;

  const long long i0 = (long long)(splitmix64(seed, 2 * (uint64_t)nd) % (uint64_t)n);
  const long long i1 = (i0 + 1 + (long long)(splitmix64(seed, 2 * (uint64_t)nd + 1) % (uint64_t)(n - 1))) % n;
  if (tid < d) {
    c[0][tid] = ld(Kr + (long long)mem[i0] * d + tid);
    c[1][tid] = ld(Kr + (long long)mem[i1] * d + tid);
  }
  for (int it = 0; it < iters; ++it) {
    __syncthreads();
    for (int j = tid; j < n; j += kSplitThreads) {
      const T* x = Kr + (long long)mem[j] * d;
      double d0 = 0.0, d1 = 0.0;
      for (int k = 0; k < d; ++k) {
        const double v = ld(x + k);
        const double t0 = __dsub_rn(v, c[0][k]), t1 = __dsub_rn(v, c[1][k]);
        d0 = __dadd_rn(d0, __dmul_rn(t0, t0));
        d1 = __dadd_rn(d1, __dmul_rn(t1, t1));
      }
      side[j] = d1 < d0 ? 1 : 0;
    }
    __syncthreads();
    double acc = 0.0;
    int ns = 0;
    const int s = tid / d, k = tid - s * d;
    if (tid < 2 * d) {
      for (int j = 0; j < n; ++j)
        if (side[j] == s) {
          acc = __dadd_rn(acc, ld(Kr + (long long)mem[j] * d + k));
          ++ns;
        }
    }
    __syncthreads();  // every thread has read c
    if (tid < 2 * d && ns > 0) c[s][k] = __ddiv_rn(acc, (double)ns);
  }
  __syncthreads();
  // left-side count; a one-sided split halves the members instead
  int z = 0;
  for (int j = tid; j < n; j += kSplitThreads) z += side[j] == 0;
  int tot;
  {
    // block sum over kSplitThreads threads through the first 8 warps' slots
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) sh[warp] = z;
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < kSplitThreads / 32; ++w) t += sh[w];
      n0_s = t;
    }
    __syncthreads();
    tot = n0_s;
  }
  int n0 = tot;
  const bool halve = n0 == 0 || n0 == n;
  if (halve) n0 = (n + 1) / 2;
  // stable partition into tmp, then back into the node's range
  int32_t* tmp = a.tmp + ko + lo;
  int zeros = 0;  // left-side members before the current chunk
  for (int base = 0; base < n; base += kSplitThreads) {
    const int j = base + tid;
    const int sj = j < n ? (halve ? (j >= n0 ? 1 : 0) : side[j]) : 1;
    const int isz = j < n && sj == 0 ? 1 : 0;
    // exclusive scan of isz over the CTA
    const int lane = tid & 31, warp = tid >> 5;
    int x = isz;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    int before = 0, chunk = 0;
    for (int w = 0; w < kSplitThreads / 32; ++w) {
      if (w < warp) before += sh[w];
      chunk += sh[w];
    }
    before += x - isz;
    if (j < n) {
      const int zb = zeros + before;       // left members before j
      const int dst = sj == 0 ? zb : n0 + (j - zb);
      tmp[dst] = mem[j];
    }
    zeros += chunk;
    __syncthreads();
  }
  __syncthreads();
  for (int j = tid; j < n; j += kSplitThreads) mem[j] = tmp[j];
  if (tid == 0) {
    const int l = a.left()[no + nd];
    a.lo()[no + l] = lo;
    a.cnt()[no + l] = n0;
    a.lo()[no + l + 1] = lo + n0;
    a.cnt()[no + l + 1] = n - n0;
  }
}

// Centroids: a warp per node, lanes over the dimensions, members in index order.
template <typename T>
__global__ void __launch_bounds__(256) c3_centroid_kernel(const RowMap m, C3Arr a, const T* __restrict__ K, int d) {
  const int row = blockIdx.y;
  const long long ko = row_key_off(m, row), no = 2 * ko;
  const int nodes = a.hdr()[(long long)row * kHdr];
  const int nd = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (nd >= nodes) return;
  const int lane = threadIdx.x & 31;
  const int lo = a.lo()[no + nd], n = a.cnt()[no + nd];
  const int32_t* mem = a.perm() + ko + lo;
  const T* Kr = K + ko * d;
  double* cr = a.cent() + (no + nd) * d;
  for (int k = lane; k < d; k += 32) {
    double s = 0.0;
    for (int j = 0; j < n; ++j) s = __dadd_rn(s, ld(Kr + (long long)mem[j] * d + k));
    cr[k] = __ddiv_rn(s, (double)n);
  }
}

// The initial frontier: nodes at depth D0 and the leaves above it, ascending.
__global__ void __launch_bounds__(kScanThreads) c3_frontier_kernel(const RowMap m, C3Arr a, int granularity) {
  __shared__ int sh[64];
  const int row = blockIdx.x;
  const int L = row_len(m, row);
  const long long no = 2 * row_key_off(m, row);
  int32_t* h = a.hdr() + (long long)row * kHdr;
  const int nodes = h[0];
  int D0 = 0;
  while (D0 < 40) {
    const double next = (double)granularity * (double)(1ll << (D0 + 1));
    if (next * next > 2.0 * (double)L * (double)L) break;
    ++D0;
  }
  int carry = 0;
  for (int base = 0; base < nodes; base += kScanThreads) {
    const int n = base + threadIdx.x;
    bool f = false;
    if (n < nodes) {
      const int dp = a.depth()[no + n];
      f = dp == D0 || (dp < D0 && a.left()[no + n] < 0);
      a.e()[no + n] = 0.0;
    }
    int tot;
    const int r = carry + scan_excl(f ? 1 : 0, &tot, sh);
    if (f) a.front()[no + r] = n;
    carry += tot;
  }
  if (threadIdx.x == 0) {
    h[1] = carry;  // A
    h[2] = 0;
  }
}

// ------------------------------------------------------------------- step --
// sigma of every frontier node: max over the query heads of the cosine
// (float64; products and sums rounded separately, every sum in dimension
// order from 0, as the oracle does). A lane takes a node; its warp copies
// the 32 nodes' centroids into shared memory 32 dimensions at a time with
// coalesced loads (eight in flight per lane; padded so the lanes' reads
// spread over the banks), and the block copies the row's query rows as
// doubles. The query norms sum q_k^2 and the centroid norm sum c_k^2 are
// each taken once (the same chains as per cosine, so the same values); the
// heads' dot products are independent chains (up to kC3Heads at a time).
// A row's blocks stride over its frontier, so the grid holds no blocks
// beyond the frontier's possible size.
constexpr int kC3ScoreWarps = 4;
constexpr int kC3Heads = 8;
constexpr int kC3QStage = 16;  // query heads staged in shared memory (more: read from global memory)
constexpr int kC3FillBatch = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kC3ScoreWarps)
    c3_score_kernel(const RowMap m, C3Arr a, const T* __restrict__ q, int G, int d, int B) {
  // [warps][32][33] centroid chunks, then [G] query norms, then [G][d] query rows if G <= kC3QStage
  extern __shared__ double c3s[];
  const int row = blockIdx.y;
  if (row_len(m, row) <= B) return;
  const long long no = 2 * row_key_off(m, row);
  const int nodes = a.hdr()[(long long)row * kHdr], A = a.hdr()[(long long)row * kHdr + 1];
  if (!kv_check(A >= 0 && A <= 2 * row_len(m, row) && nodes <= 2 * row_len(m, row))) return;
  const int per_blk = 32 * kC3ScoreWarps;
  if (blockIdx.x * per_blk >= A) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double* cs = c3s + (size_t)warp * 32 * 33;
  double* qn = c3s + (size_t)kC3ScoreWarps * 32 * 33;
  double* qs = qn + G;
  const T* qr = q + (long long)row * G * d;
  const bool q_staged = G <= kC3QStage;
  if (q_staged)
    for (int k = threadIdx.x; k < G * d; k += per_blk) qs[k] = ld(qr + k);
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += per_blk) {
    double aa = 0.0;
    for (int k = 0; k < d; ++k) {
      const double x = q_staged ? qs[g * d + k] : ld(qr + (long long)g * d + k);
      aa = __dadd_rn(aa, __dmul_rn(x, x));
    }
    qn[g] = aa;
  }
  __syncthreads();
  for (int i0 = blockIdx.x * per_blk; i0 < A; i0 += gridDim.x * per_blk) {
    const int wi0 = i0 + warp * 32;
    if (wi0 >= A) break;
    const int i = wi0 + lane;
    const int nw = min(32, A - wi0);  // nodes of this warp
    int my_node = i < A ? a.front()[no + i] : 0;
    if (!kv_check(my_node >= 0 && my_node < nodes)) my_node = 0;
    double bb = 0.0, best = -INFINITY;
    for (int g0 = 0; g0 < G; g0 += kC3Heads) {
      double ab[kC3Heads];
#pragma unroll
      for (int t = 0; t < kC3Heads; ++t) ab[t] = 0.0;
      for (int k0 = 0; k0 < d; k0 += 32) {
        __syncwarp();
        for (int n0 = 0; n0 < nw; n0 += kC3FillBatch) {  // node n's dimensions k0 .. k0 + 31, one per lane
          double v[kC3FillBatch];
#pragma unroll
          for (int u = 0; u < kC3FillBatch; ++u) {
            const int node = __shfl_sync(0xffffffffu, my_node, (n0 + u) & 31);
            v[u] = n0 + u < nw ? a.cent()[(no + node) * d + k0 + lane] : 0.0;
          }
#pragma unroll
          for (int u = 0; u < kC3FillBatch; ++u)
            if (n0 + u < nw) cs[(n0 + u) * 33 + lane] = v[u];
        }
        __syncwarp();
        if (i < A) {
          for (int kk = 0; kk < 32; ++kk) {
            const int k = k0 + kk;
            const double yk = cs[lane * 33 + kk];
            if (g0 == 0) bb = __dadd_rn(bb, __dmul_rn(yk, yk));
#pragma unroll
            for (int t = 0; t < kC3Heads; ++t)
              if (g0 + t < G) {
                const double x = q_staged ? qs[(g0 + t) * d + k] : ld(qr + (long long)(g0 + t) * d + k);
                ab[t] = __dadd_rn(ab[t], __dmul_rn(x, yk));
              }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kC3Heads; ++t)
        if (g0 + t < G) {
          const double aa = qn[g0 + t];
          const double c = (aa == 0.0 || bb == 0.0) ? 0.0 : __ddiv_rn(ab[t], __dmul_rn(__dsqrt_rn(aa), __dsqrt_rn(bb)));
          if (c > best) best = c;
        }
    }
    if (i < A) a.sigma()[no + i] = best;
  }
}

// Order key of a frontier entry: larger sigma first, then the lower node id.
__device__ __forceinline__ uint64_t sigma_key(double s) {
  uint64_t u = (uint64_t)__double_as_longlong(s);
  if (u == 0x8000000000000000ull) u = 0;  // -0 == +0
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// The retrieved positions of a row: clusters in key order until B members.
__global__ void __launch_bounds__(kScanThreads) c3_select_kernel(const RowMap m, C3Arr a, int B) {
  __shared__ int hist[256];
  __shared__ int sh[64];
  __shared__ unsigned long long thi_s;
  __shared__ unsigned int tlo_s;
  __shared__ int need_s;
  const int row = blockIdx.x;
  const int L = row_len(m, row);
  const long long ko = row_key_off(m, row), no = 2 * ko;
  int32_t* h = a.hdr() + (long long)row * kHdr;
  int32_t* sel = a.sel() + ko;
  if (L <= B) {  // bypass: every key
    for (int j = threadIdx.x; j < L; j += kScanThreads) sel[j] = j;
    if (threadIdx.x == 0) h[2] = L;
    return;
  }
  const int nodes = h[0], A = h[1];
  const int32_t* fr = a.front() + no;
  const double* sg = a.sigma() + no;
  if (kDebugChecks) {  // the row's frontier: its size and node ids, and each node's members
    bool bad = !kv_check(A >= 0 && A <= 2 * L && nodes <= 2 * L);
    for (int i = threadIdx.x; !bad && i < A; i += kScanThreads) {
      const int n = fr[i];
      bad = !kv_check(n >= 0 && n < nodes && a.lo()[no + n] >= 0 && a.cnt()[no + n] >= 0 &&
                      a.lo()[no + n] + a.cnt()[no + n] <= L);
    }
    if (__syncthreads_or(bad)) return;
  }
  if (threadIdx.x == 0) {
    thi_s = 0;
    tlo_s = 0;
    need_s = B;
  }
  // weighted radix select over the 96-bit keys (sigma key, ~node id), 8 bits a
  // round; a thread keeps its first kC3SelReg entries in registers, and warp 0
  // finds each round's bin (the entries' weights, the clusters' sizes, add up
  // to L > B, so the bins always hold `need`)
  uint64_t khi[kC3SelReg];
  uint32_t klo[kC3SelReg];
  int kcnt[kC3SelReg];
#pragma unroll
  for (int u = 0; u < kC3SelReg; ++u) {
    const int i = threadIdx.x + u * kScanThreads;
    khi[u] = 0;
    klo[u] = 0;
    kcnt[u] = 0;
    if (i < A) {
      const int n = fr[i];
      khi[u] = sigma_key(sg[i]);
      klo[u] = ~(uint32_t)n;
      kcnt[u] = a.cnt()[no + n];
    }
  }
  for (int round = 0; round < 12; ++round) {
    for (int i = threadIdx.x; i < 256; i += kScanThreads) hist[i] = 0;
    __syncthreads();
    const unsigned long long phi = thi_s;
    const unsigned int plo = tlo_s;
    auto count = [&](uint64_t hi, uint32_t lo, int c) {
      bool match;
      int digit;
      if (round < 8) {
        const int sh_hi = 56 - 8 * round;
        const uint64_t mask = round == 0 ? 0ull : (~0ull << (sh_hi + 8));
        match = (hi & mask) == (phi & mask);
        digit = (int)((hi >> sh_hi) & 255u);
      } else {
        const int sh_lo = 24 - 8 * (round - 8);
        const uint32_t mask = round == 8 ? 0u : (~0u << (sh_lo + 8));
        match = hi == phi && (lo & mask) == (plo & mask);
        digit = (int)((lo >> sh_lo) & 255u);
      }
      if (match) atomicAdd(&hist[digit], c);
    };
#pragma unroll
    for (int u = 0; u < kC3SelReg; ++u)
      if (threadIdx.x + u * kScanThreads < A) count(khi[u], klo[u], kcnt[u]);
    for (int i = threadIdx.x + kC3SelReg * kScanThreads; i < A; i += kScanThreads)
      count(sigma_key(sg[i]), ~(uint32_t)fr[i], a.cnt()[no + fr[i]]);
    __syncthreads();
    if (threadIdx.x < 32) {
      int need = need_s;
      const int dg = top_bin(hist, need);
      if (threadIdx.x == 0) {
        need_s = need;
        if (round < 8) thi_s = phi | ((unsigned long long)dg << (56 - 8 * round));
        else tlo_s = plo | ((unsigned int)dg << (24 - 8 * (round - 8)));
      }
    }
    __syncthreads();
  }
  const uint64_t thi = thi_s;
  const uint32_t tlo = tlo_s;
  const int need = need_s;  // members the threshold cluster gives
  for (int j = threadIdx.x; j < L; j += kScanThreads) a.taken[ko + j] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < A; i += kScanThreads) {
    const uint64_t hi = sigma_key(sg[i]);
    const uint32_t lo = ~(uint32_t)fr[i];
    const int n = fr[i];
    int take = 0;
    if (hi > thi || (hi == thi && lo > tlo)) take = a.cnt()[no + n];
    else if (hi == thi && lo == tlo) take = need;
    const int32_t* mem = a.perm() + ko + a.lo()[no + n];
    for (int j = 0; j < take; ++j)
      if (kv_check(mem[j] >= 0 && mem[j] < L)) a.taken[ko + mem[j]] = 1;
  }
  __syncthreads();
  int carry = 0;
  for (int base = 0; base < L; base += kScanThreads) {
    const int j = base + threadIdx.x;
    const bool t = j < L && a.taken[ko + j];
    int tot;
    const int r = carry + scan_excl(t ? 1 : 0, &tot, sh);
    if (t) sel[r] = j;
    carry += tot;
  }
  if (threadIdx.x == 0) h[2] = carry;
}

template <typename T>
__device__ __forceinline__ void st_out(T* p, float v);
template <>
__device__ __forceinline__ void st_out<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;

// Up to four consecutive elements of a K or V row as float32.
template <typename T>
__device__ __forceinline__ void ld4(const T* p, int n, float (&v)[4]);
template <>
__device__ __forceinline__ void ld4<float>(const float* p, int n, float (&v)[4]) {
  if (n == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = v[3] = 0.f;
  }
}
template <>
__device__ __forceinline__ void ld4<__nv_bfloat16>(const __nv_bfloat16* p, int n, float (&v)[4]) {
  if (n == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    v[0] = a.x; v[1] = a.y; v[2] = v[3] = 0.f;
  }
}

// Exact attention of one query head over the retrieved keys (float32): a warp
// per key for the logits (each lane d/32 consecutive elements), then p V with
// the keys split over the warps (lanes over the dimensions) and the warps'
// partial sums added in warp order.
template <typename T>
__global__ void __launch_bounds__(kAttnThreads)
    c3_attn_kernel(const RowMap m, C3Arr a, const T* __restrict__ K, const T* __restrict__ V,
                   const T* __restrict__ q, T* __restrict__ out, int G, int d, int B) {
  extern __shared__ float dyn_s[];  // logits [B], then the retrieved positions [B]
  float* lg = dyn_s;
  int* sel_s = reinterpret_cast<int*>(dyn_s + B);
  __shared__ float qv[128];
  __shared__ float red[32];
  __shared__ float po[kAttnWarps][128];
  const int row = blockIdx.x, g = blockIdx.y;
  const long long ko = row_key_off(m, row);
  const int n = min(a.hdr()[(long long)row * kHdr + 2], B);  // the select kernel retrieves at most B
  const int32_t* sel = a.sel() + ko;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = d / 32;  // elements per lane: 2 or 4
  const T* qr = q + ((long long)row * G + g) * d;
  for (int k = threadIdx.x; k < d; k += kAttnThreads) qv[k] = (float)ld(qr + k);
  for (int i = threadIdx.x; i < n; i += kAttnThreads) {
    const int p = sel[i];
    sel_s[i] = kv_check(p >= 0 && p < row_len(m, row)) ? p : 0;
  }
  __syncthreads();
  const float scale = rsqrtf((float)d);
  float qa[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) qa[t] = t < per ? qv[lane * per + t] : 0.f;
  for (int i = warp; i < n; i += kAttnWarps) {
    float kv4[4];
    ld4(K + (ko + sel_s[i]) * d + lane * per, per, kv4);
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) s = fmaf(qa[t], kv4[t], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) lg[i] = s * scale;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < n; i += kAttnThreads) mx = fmaxf(mx, lg[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < kAttnWarps; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int i = threadIdx.x; i < n; i += kAttnThreads) {
    const float p = __expf(lg[i] - mx);
    lg[i] = p;
    sum += p;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < kAttnWarps; ++w) sum += red[w];
  // p V: warp w takes the keys [w n / 8, (w + 1) n / 8), lane the elements lane * per ...
  {
    const int i0 = (int)((long long)n * warp / kAttnWarps), i1 = (int)((long long)n * (warp + 1) / kAttnWarps);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int i = i0; i < i1; ++i) {
      float vv[4];
      ld4(V + (ko + sel_s[i]) * d + lane * per, per, vv);
      const float p = lg[i];
#pragma unroll
      for (int t = 0; t < 4; ++t) acc[t] = fmaf(p, vv[t], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < per) po[warp][lane * per + t] = acc[t];
  }
  __syncthreads();
  T* orow = out + ((long long)row * G + g) * d;
  for (int k = threadIdx.x; k < d; k += kAttnThreads) {
    float acc = 0.f;
    for (int w = 0; w < kAttnWarps; ++w) acc += po[w][k];
    st_out(orow + k, acc / sum);
  }
}

// (larger value, then lower id) wins when mx; (smaller value, then lower id) otherwise
__device__ __forceinline__ bool wins(double v, int i, double bv, int bi, bool mx) {
  if (i < 0) return false;
  if (bi < 0) return true;
  if (mx ? v > bv : v < bv) return true;
  return v == bv && i < bi;
}

__device__ void block_pick(double& v, int& i, bool mx, double* shv, int* shi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_down_sync(0xffffffffu, v, o);
    const int oi = __shfl_down_sync(0xffffffffu, i, o);
    if (wins(ov, oi, v, i, mx)) {
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
    v = shv[lane];
    i = shi[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_down_sync(0xffffffffu, v, o);
      const int oi = __shfl_down_sync(0xffffffffu, i, o);
      if (wins(ov, oi, v, i, mx)) {
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

// EMA of the frontier, R split/merge exchanges, frontier compaction.
__global__ void __launch_bounds__(kScanThreads)
    c3_update_kernel(const RowMap m, C3Arr a, int B, double lambda, int R) {
  __shared__ int sh[64];
  __shared__ double shv[32];
  __shared__ int shi[32];
  const int row = blockIdx.x;
  if (row_len(m, row) <= B) return;
  const long long no = 2 * row_key_off(m, row);
  int32_t* h = a.hdr() + (long long)row * kHdr;
  const int nodes = h[0], A = h[1];
  int32_t* fr = a.front() + no;
  if (kDebugChecks) {  // the row's frontier: its size and node ids
    const int L = row_len(m, row);
    bool bad = !kv_check(A >= 0 && A <= 2 * L && nodes <= 2 * L);
    for (int i = threadIdx.x; !bad && i < A; i += kScanThreads) bad = !kv_check(fr[i] >= 0 && fr[i] < nodes);
    if (__syncthreads_or(bad)) return;
  }
  double* e = a.e() + no;
  const int32_t* left = a.left() + no;
  uint8_t* on = a.on + no;
  uint8_t* fresh = a.fresh + no;
  const double keep = __dsub_rn(1.0, lambda);
  for (int i = threadIdx.x; i < A; i += kScanThreads)
    e[fr[i]] = __dadd_rn(__dmul_rn(lambda, e[fr[i]]), __dmul_rn(keep, a.sigma()[no + i]));
  for (int n = threadIdx.x; n < nodes; n += kScanThreads) on[n] = fresh[n] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < A; i += kScanThreads) on[fr[i]] = 1;
  __syncthreads();
  // Every candidate of an exchange is a node of the step's starting frontier
  // that is still on and was not made in this step (nodes made in the step are
  // fresh), so both searches walk the frontier list instead of every node; the
  // winners (ties to the lower node id) are the same.
  const int32_t* parent = a.parent + no;
  for (int r = 0; r < R; ++r) {
    double sv = 0.0;
    int s = -1;
    for (int i = threadIdx.x; i < A; i += kScanThreads) {
      const int n = fr[i];
      if (on[n] && !fresh[n] && left[n] >= 0 && wins(e[n], n, sv, s, true)) {
        sv = e[n];
        s = n;
      }
    }
    block_pick(sv, s, true, shv, shi);
    if (s < 0) break;
    // merge: the parent of two siblings still on the frontier (x its left child)
    double pv = 0.0;
    int p = -1;
    for (int i = threadIdx.x; i < A; i += kScanThreads) {
      const int x = fr[i];
      const int n = parent[x];
      if (n < 0 || left[n] != x) continue;
      const int y = x + 1;
      if (!on[x] || !on[y] || fresh[x] || fresh[y] || x == s || y == s) continue;
      const double v = e[x] > e[y] ? e[x] : e[y];
      if (wins(v, n, pv, p, false)) {
        pv = v;
        p = n;
      }
    }
    block_pick(pv, p, false, shv, shi);
    if (p < 0) break;
    if (threadIdx.x == 0) {
      const int c = left[s];
      on[s] = 0;
      on[c] = on[c + 1] = 1;
      fresh[c] = fresh[c + 1] = 1;
      e[c] = e[c + 1] = e[s];
      on[left[p]] = on[left[p] + 1] = 0;
      on[p] = 1;
      fresh[p] = 1;
      e[p] = pv;
    }
    __syncthreads();
  }
  int carry = 0;
  for (int base = 0; base < nodes; base += kScanThreads) {
    const int n = base + threadIdx.x;
    const bool f = n < nodes && on[n];
    int tot;
    const int rr = carry + scan_excl(f ? 1 : 0, &tot, sh);
    if (f) fr[rr] = n;
    carry += tot;
  }
}

// ------------------------------------------------------------------- host --
bool c3_params_ok(const kv_c3_params* p) {
  if (!p) return false;
  if (p->leaf_max < 1 || p->iters < 1 || p->iters > 64 || p->granularity < 4) return false;
  if (p->budget < 1 || p->budget > KV_C3_MAX_BUDGET || p->exchanges < 0 || p->exchanges > 64) return false;
  return p->lambda >= 0.0 && p->lambda <= 1.0;
}

int c3_map(const kv_shape* sh, const int32_t* L, int32_t n_seq, RowMap& m) {
  if (!sh || !L || n_seq < 1 || n_seq > KV_MAX_SEQ) return KV_ERR_ARG;
  if (sh->n_layers < 1 || sh->n_kv_heads < 1 || sh->group < 1 || sh->group > 16) return KV_ERR_ARG;
  if (sh->head_dim != 64 && sh->head_dim != 128) return KV_ERR_ARG;
  if (sh->dtype != KV_BF16 && sh->dtype != KV_F32) return KV_ERR_ARG;
  std::memset(&m, 0, sizeof(m));
  m.n_seq = n_seq;
  m.rows_per_seq = sh->n_layers * sh->n_kv_heads;
  m.n_rows = n_seq * m.rows_per_seq;
  long long key = 0;
  for (int s = 0; s < n_seq; ++s) {
    if (L[s] < 1 || L[s] > KV_MAX_L) return KV_ERR_UNSUPPORTED_L;
    m.L[s] = L[s];
    m.key_off[s] = key;
    key += (long long)m.rows_per_seq * L[s];
  }
  m.key_off[n_seq] = key;
  return KV_OK;
}

int max_len(const RowMap& m) {
  int x = 0;
  for (int s = 0; s < m.n_seq; ++s) x = std::max(x, m.L[s]);
  return x;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" {

int kv_c3_index_layout(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p,
                       kv_c3_layout* out) {
  RowMap m;
  const int st = c3_map(shape, L, n_seq, m);
  if (st != KV_OK) return st;
  if (!c3_params_ok(p) || !out) return KV_ERR_ARG;
  C3Scratch S;
  layout_of(m.key_off[n_seq], m.n_rows, shape->head_dim, *out, S);
  return KV_OK;
}

int kv_c3_build(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p, const void* K,
                void* index, void* stream) {
  RowMap m;
  int st = c3_map(shape, L, n_seq, m);
  if (st != KV_OK) return st;
  if (!c3_params_ok(p) || !K || !index || (reinterpret_cast<uintptr_t>(index) & 255u)) return KV_ERR_ARG;
  kv_c3_layout lay;
  C3Scratch S;
  layout_of(m.key_off[n_seq], m.n_rows, shape->head_dim, lay, S);
  C3Arr a = arrays_of(index, lay, S);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int d = shape->head_dim;
  const bool bf = shape->dtype == KV_BF16;
  c3_init_kernel<<<m.n_rows, 256, 0, cs>>>(m, a);
  int32_t host_count = 0;  // pageable: the copy completes before the synchronise returns
  st = KV_OK;
  for (int level = 0; level < (1 << 20); ++level) {
    if (cudaMemsetAsync(a.count, 0, sizeof(int32_t), cs) != cudaSuccess) {
      st = KV_ERR_CUDA;
      break;
    }
    c3_plan_kernel<<<m.n_rows, kScanThreads, 0, cs>>>(m, a, p->leaf_max);
    if (cudaMemcpyAsync(&host_count, a.count, sizeof(int32_t), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess) {
      st = KV_ERR_CUDA;
      break;
    }
    const int tasks = host_count;
    if (tasks == 0) break;
    if (bf)
      c3_split_kernel<__nv_bfloat16><<<tasks, kSplitThreads, 0, cs>>>(m, a, static_cast<const __nv_bfloat16*>(K), d,
                                                                     p->iters, p->seed);
    else
      c3_split_kernel<float><<<tasks, kSplitThreads, 0, cs>>>(m, a, static_cast<const float*>(K), d, p->iters,
                                                              p->seed);
  }
  if (st != KV_OK) return st;
  const int Lmax = max_len(m);
  const dim3 cg((2 * Lmax + 7) / 8, m.n_rows);
  if (bf)
    c3_centroid_kernel<__nv_bfloat16><<<cg, 256, 0, cs>>>(m, a, static_cast<const __nv_bfloat16*>(K), d);
  else
    c3_centroid_kernel<float><<<cg, 256, 0, cs>>>(m, a, static_cast<const float*>(K), d);
  c3_frontier_kernel<<<m.n_rows, kScanThreads, 0, cs>>>(m, a, p->granularity);
  return cuda_status(cudaGetLastError());
}

int kv_c3_step(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p, const void* K,
               const void* V, const void* q, void* index, void* out, void* stream) {
  RowMap m;
  const int st = c3_map(shape, L, n_seq, m);
  if (st != KV_OK) return st;
  if (!c3_params_ok(p) || !K || !V || !q || !index || !out || (reinterpret_cast<uintptr_t>(index) & 255u))
    return KV_ERR_ARG;
  kv_c3_layout lay;
  C3Scratch S;
  layout_of(m.key_off[n_seq], m.n_rows, shape->head_dim, lay, S);
  C3Arr a = arrays_of(index, lay, S);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int d = shape->head_dim, G = shape->group, B = p->budget;
  const int Lmax = max_len(m);
  // blocks per row: the frontier's largest possible size (2 L nodes), capped so
  // that the grid is about four waves of resident blocks; the blocks stride
  const int per_blk = 32 * kC3ScoreWarps;
  const size_t score_smem =
      ((G <= kC3QStage ? (size_t)G * d : 0) + (size_t)G + (size_t)kC3ScoreWarps * 32 * 33) * sizeof(double);
  const int resident = sm_count() * (int)std::max<size_t>(1, (228u << 10) / (score_smem + 1024));
  const int sx = std::max(1, std::min((2 * Lmax + per_blk - 1) / per_blk, (4 * resident + m.n_rows - 1) / m.n_rows));
  const dim3 sgrid(sx, m.n_rows);
  const size_t attn_smem = 2 * (size_t)B * sizeof(float);  // logits and retrieved positions
  if (shape->dtype == KV_BF16) {
    using T = __nv_bfloat16;
    if (cudaFuncSetAttribute(c3_score_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)score_smem) !=
        cudaSuccess)
      return KV_ERR_CUDA;
    c3_score_kernel<T><<<sgrid, 32 * kC3ScoreWarps, score_smem, cs>>>(m, a, static_cast<const T*>(q), G, d, B);
    c3_select_kernel<<<m.n_rows, kScanThreads, 0, cs>>>(m, a, B);
    if (cudaFuncSetAttribute(c3_attn_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn_smem) !=
        cudaSuccess)
      return KV_ERR_CUDA;
    c3_attn_kernel<T><<<dim3(m.n_rows, G), kAttnThreads, attn_smem, cs>>>(
        m, a, static_cast<const T*>(K), static_cast<const T*>(V), static_cast<const T*>(q), static_cast<T*>(out), G,
        d, B);
  } else {
    using T = float;
    if (cudaFuncSetAttribute(c3_score_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)score_smem) !=
        cudaSuccess)
      return KV_ERR_CUDA;
    c3_score_kernel<T><<<sgrid, 32 * kC3ScoreWarps, score_smem, cs>>>(m, a, static_cast<const T*>(q), G, d, B);
    c3_select_kernel<<<m.n_rows, kScanThreads, 0, cs>>>(m, a, B);
    if (cudaFuncSetAttribute(c3_attn_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn_smem) !=
        cudaSuccess)
      return KV_ERR_CUDA;
    c3_attn_kernel<T><<<dim3(m.n_rows, G), kAttnThreads, attn_smem, cs>>>(
        m, a, static_cast<const T*>(K), static_cast<const T*>(V), static_cast<const T*>(q), static_cast<T*>(out), G,
        d, B);
  }
  c3_update_kernel<<<m.n_rows, kScanThreads, 0, cs>>>(m, a, B, p->lambda, p->exchanges);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
