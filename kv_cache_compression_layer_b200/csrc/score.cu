// kv_score: observation-window importance scores (AudioKV blog §1.2, the raw
// importance scores that Spectral Score Smoothing later smooths):
//   s_j = sum_{r<R} softmax_j(q_r . K_j / sqrt(d)),  R = g * w window rows.
//
// bf16 path (tcgen05 + TMEM + TMA), two passes over K with a tiny merge:
//   pass 1  D[r][j] = Q K_tile^T on the tensor core (M = 128 window rows per
//           half, N = 128 keys); the epilogue turns each row of the tile into
//           (tile max m, sum of exp2((x - m) c)) partials.
//   merge   per (row, r): lse2_r = log2 of the softmax denominator (c = log2 e
//           / sqrt d units), from the tile partials.
//   pass 2  D[j][r] = K_tile Q^T (M = 128 keys, N = R); each epilogue thread
//           owns one key and sums exp2(x c - lse2_r) over the R window rows.
// Both passes are persistent (one CTA per SM, contiguous runs of tiles) and
// warp-specialised: warp 0 issues TMA loads of Q and a 4-stage ring of K
// tiles, warp 1 issues tcgen05.mma into a double-buffered TMEM accumulator,
// warps 2-17 read TMEM with tcgen05.ld and do the softmax arithmetic: four
// groups of four warps (one warp per TMEM lane quarter), two groups per
// accumulator buffer. In pass 1 the two groups of a buffer take the two
// halves of the window rows (a warp whose 32 rows all lie at or beyond R does
// nothing); in pass 2 they take the two halves of the R columns, and the
// first half hands its per-key sums to the second through shared memory
// (added in a fixed order). The exponentials are the binding unit, so the
// epilogue reads TMEM in 32-column chunks and overlaps each chunk's load with
// the previous chunk's arithmetic; pass 1 keeps a running maximum per row.
//
// fp32 path (fp32 inputs): the same three steps on CUDA cores (FFMA), since
// a tf32 contraction would not meet the fp32 tolerance.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace kvc {
namespace {

constexpr int kStages = 4;
constexpr int kQRows = 256;
constexpr int kEpiWarps = 16;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kQChunkBytes = kQRows * 128;      // 256 rows x 64 bf16
constexpr int kKChunkBytes = kTileKeys * 128;   // 128 keys x 64 bf16
constexpr int kKStageBytes = 2 * kKChunkBytes;  // d <= 128
constexpr int kSmemQ = 0;
constexpr int kSmemK = 2 * kQChunkBytes;
constexpr int kSmemBar = kSmemK + kStages * kKStageBytes;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 1;
constexpr int kSmemMisc = kSmemBar + kNumBars * 8;
constexpr int kSmemPart = kSmemMisc + 16;                  // pass 2: [buffer][parity][128 keys] float
// pass 2: [epilogue warp][128 columns] float, read as float4 (16-byte aligned)
constexpr int kSmemLse = (kSmemPart + 2 * 2 * kTileKeys * 4 + 127) & ~127;
static_assert(kSmemLse % 16 == 0, "float4 reads of the staged lse2");
constexpr int kSmemTotal = kSmemLse + kEpiWarps * 128 * 4;
constexpr int kSmemAlloc = kSmemTotal + 1024;  // slack for 1024-byte alignment

struct TcArgs {
  RowMap map;
  int R;      // valid window rows
  int n2;     // pass-2 MMA N: R rounded up to 16
  int total_tiles;
  float c;    // log2(e) / sqrt(d)
  int Rs;     // row stride of lse2: R rounded up to 4 (16-byte rows)
  float2* partial;     // pass 1 out: [total_tiles][R] (tile max, tile sum)
  const float* lse2;   // pass 2 in:  [rows][Rs]
  float* s;            // pass 2 out: [sum L]
  int* status;
  unsigned long long limit_ns;
};

// Walks a CTA's contiguous run of scoring tiles in order: the row, the tile
// in the row, its valid keys and the row's first key, advanced without a
// search (the sequences' rows and keys are laid out one after another).
struct TileIter {
  int row, tile, tpr, L;
  long long key0;  // first key of the row
  __device__ __forceinline__ void init(const RowMap& m, int u) {
    int s = 0;
    while (s + 1 < m.n_seq && m.tile_off[s + 1] <= u) ++s;
    L = m.L[s];
    tpr = (L + kTileKeys - 1) / kTileKeys;
    const int local = u - m.tile_off[s];
    row = s * m.rows_per_seq + local / tpr;
    tile = local % tpr;
    key0 = m.key_off[s] + (long long)(row - s * m.rows_per_seq) * L;
  }
  __device__ __forceinline__ void next(const RowMap& m) {
    if (++tile < tpr) return;
    tile = 0;
    key0 += L;
    ++row;
    if (row % m.rows_per_seq == 0 && row < m.n_rows) {  // the next sequence's first row
      L = m.L[row / m.rows_per_seq];
      tpr = (L + kTileKeys - 1) / kTileKeys;
    }
  }
  __device__ __forceinline__ int nvalid() const { return min(kTileKeys, L - tile * kTileKeys); }
};

// Epilogue warps with work per accumulator buffer: pass 1, the (row half,
// lane quarter) pairs holding some row < R; pass 2, four per column half that
// holds a 32-column chunk (the first half is empty when there is one chunk).
template <int PASS>
__host__ __device__ constexpr int epi_active_warps(int R, int n2) {
  if (PASS == 1) {
    int n = 0;
    for (int h = 0; h < 2; ++h)
      for (int q = 0; q < 4; ++q) n += h * 128 + q * 32 < R ? 1 : 0;
    return n;
  }
  return ((n2 + 31) / 32) / 2 > 0 ? 8 : 4;
}

template <int PASS, int NK>  // NK: 64-column chunks of d
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sK = smem + kSmemK;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* full_k = bars;
  uint64_t* empty_k = bars + kStages;
  uint64_t* q_full = bars + 2 * kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* acc_full = q_full + 2;
  uint64_t* acc_empty = q_full + 4;
  uint64_t* drain = q_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int u0 = (int)((long long)a.total_tiles * blockIdx.x / G);
  const int u1 = (int)((long long)a.total_tiles * (blockIdx.x + 1) / G);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&empty_k[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], epi_active_warps<PASS>(a.R, a.n2));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, a.status, a.limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      TileIter ti;
      if (u0 < u1) ti.init(a.map, u0);
      int cur_row = -1, st = 0;
      uint32_t qe_phase = 0, kphase = 0;  // kphase: the parity of the stage ring's current round
      bool have_q = false;
      bool k_issued[kStages] = {false, false, false, false};
      uint32_t k_parity[kStages] = {0, 0, 0, 0};
      uint32_t q_parity = 0;
      bool aborted = false;
      for (int u = u0; u < u1; ++u, ti.next(a.map)) {
        const int row = ti.row;
        if (row != cur_row) {
          if (have_q) {
            if (!wait_bounded(q_empty, qe_phase, g)) { aborted = true; break; }
            qe_phase ^= 1;
            q_parity ^= 1;
          }
          have_q = true;
          cur_row = row;
          mbar_arrive_expect_tx(q_full, NK * kQChunkBytes);
#pragma unroll
          for (int c = 0; c < NK; ++c) tma_load_2d(sQ + c * kQChunkBytes, &tmQ, q_full, c * 64, row * a.R);
        }
        // the stage's previous round has been consumed (from the second round on)
        if (u - u0 >= kStages && !wait_bounded(&empty_k[st], kphase ^ 1, g)) { aborted = true; break; }
        mbar_arrive_expect_tx(&full_k[st], NK * kKChunkBytes);
        const int key0 = (int)(ti.key0 + (long long)ti.tile * kTileKeys);
#pragma unroll
        for (int c = 0; c < NK; ++c)
          tma_load_2d(sK + st * kKStageBytes + c * kKChunkBytes, &tmK, &full_k[st], c * 64, key0);
#pragma unroll
        for (int z = 0; z < kStages; ++z)  // constant indices: the arrays stay in registers
          if (z == st) {
            k_issued[z] = true;
            k_parity[z] = kphase;
          }
        if (++st == kStages) {
          st = 0;
          kphase ^= 1;
        }
      }
      // let every copy issued land before the CTA's shared memory goes away (after
      // a normal run they all have; after an abort raised anywhere some may not)
      (void)aborted;
#pragma unroll
      for (int st = 0; st < kStages; ++st)
        if (k_issued[st]) wait_drain(&full_k[st], k_parity[st]);
      if (have_q) wait_drain(q_full, q_parity);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // One thread issues every MMA and shares its scheduler with four busy
      // epilogue warps, so its loop is kept short: no search for the tile's row,
      // and the operand descriptors are fixed ones plus constant offsets (the
      // 14-bit address field holds (address >> 4), which an added offset inside
      // shared memory never carries out of).
      TileIter ti;
      if (u0 < u1) ti.init(a.map, u0);
      int cur_row = -1, st = 0;
      uint32_t qf_phase = 0, kphase = 0;
      const uint64_t qdesc = sw128_kmajor_desc(smem_u32(sQ));
      const uint64_t kdesc = sw128_kmajor_desc(smem_u32(sK));
      const uint32_t idesc = PASS == 1 ? idesc_bf16_f32(128, 128) : idesc_bf16_f32(128, a.n2);
      const bool upper = a.R > 128;  // pass 1: window rows in the second 128-row half
      for (int u = u0, it = 0; u < u1; ++u, ++it) {
        const int row = ti.row;
        if (row != cur_row) {
          if (!wait_bounded(q_full, qf_phase, g)) break;
          qf_phase ^= 1;
          cur_row = row;
        }
        if (!wait_bounded(&full_k[st], kphase, g)) break;
        const int acc = it & 1;
        if (it >= 2 && !wait_bounded(&acc_empty[acc], ((it >> 1) - 1) & 1, g)) break;
        tc_fence_after();
        const uint32_t d_base = tmem + acc * 256;
        const uint64_t kd = kdesc + (uint64_t)((st * kKStageBytes) >> 4);
        uint64_t qd = qdesc;
        asm volatile("" : "+l"(qd));  // offsets added per tile, not all held across the loop
        if (PASS == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h == 0 || upper) {
#pragma unroll
              for (int kk = 0; kk < NK * 4; ++kk)
                tc_mma_bf16(d_base + h * 128,
                            qd + (uint64_t)(((kk >> 2) * kQChunkBytes + h * 128 * 128 + (kk & 3) * 32) >> 4),
                            kd + (uint64_t)(((kk >> 2) * kKChunkBytes + (kk & 3) * 32) >> 4), idesc, kk > 0);
            }
        } else {
#pragma unroll
          for (int kk = 0; kk < NK * 4; ++kk)
            tc_mma_bf16(d_base, kd + (uint64_t)(((kk >> 2) * kKChunkBytes + (kk & 3) * 32) >> 4),
                        qd + (uint64_t)(((kk >> 2) * kQChunkBytes + (kk & 3) * 32) >> 4), idesc, kk > 0);
        }
        tc_commit(&empty_k[st]);
        tc_commit(&acc_full[acc]);
        ti.next(a.map);
        if (u + 1 >= u1 || ti.row != row) tc_commit(q_empty);  // the row's last tile: Q may be replaced
        if (++st == kStages) {
          st = 0;
          kphase ^= 1;
        }
      }
      // every issued MMA has finished before TMEM is released
      tc_commit(drain);
      wait_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int e = warp - 2;
    const int quarter = warp & 3;         // TMEM lanes [32 quarter, 32 quarter + 32)
    const int bf = (e >> 2) >> 1;         // accumulator buffer of this warp's group
    const int half = (e >> 2) & 1;        // pass 1: rows [128 half, ...); pass 2: column half
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const int nc = (a.n2 + 31) / 32;      // pass 2: 32-column chunks of the accumulator
    const int c_lo = half ? nc / 2 : 0, c_hi = half ? nc : nc / 2;
    const bool active = PASS == 1 ? half * 128 + quarter * 32 < a.R : c_lo < c_hi;
    const bool pair = PASS == 2 && nc / 2 > 0;  // both column halves active: hand-off through shared memory
    const int n_pair = 32 * epi_active_warps<PASS>(a.R, a.n2);  // pass 2: the buffer's threads
    float* part = reinterpret_cast<float*>(smem + kSmemPart);
    // pass 2: this warp's columns of the current row's lse2, staged once per row
    float* lse_s = reinterpret_cast<float*>(smem + kSmemLse) + e * 128;
    int lrow = -1;
    TileIter ti;  // pass 1; pass 2 looks each tile up (its epilogue has no registers to spare)
    if (PASS == 1 && u0 + bf < u1) ti.init(a.map, u0 + bf);
    for (int u = u0 + bf; active && u < u1; u += 2) {
      const int it = u - u0;
      int row, tile, nvalid;
      if (PASS == 1) {
        row = ti.row;
        tile = ti.tile;
        nvalid = ti.nvalid();
        ti.next(a.map);  // this buffer's next tile is two on
        ti.next(a.map);
      } else {
        tile_to_row(a.map, u, row, tile);
        nvalid = min(kTileKeys, row_len(a.map, row) - tile * kTileKeys);
      }
      if (PASS == 2 && row != lrow) {
        __syncwarp();  // the previous row's values are no longer read
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int col = (c_lo + k) * 32 + lane;
          if (c_lo + k < c_hi) lse_s[k * 32 + lane] = col < a.R ? __ldg(a.lse2 + (long long)row * a.Rs + col) : 0.f;
        }
        __syncwarp();
        lrow = row;
      }
      // the warp (pass 2: the buffer's warps) leave together: tensor-memory loads are
      // warp-wide and the column halves meet at a barrier
      bool ok = __all_sync(0xffffffffu, wait_bounded(&acc_full[bf], (it >> 1) & 1, g));
      if (pair) ok = named_bar_and(1 + bf, n_pair, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem + lane_addr + bf * 256;
      float xa[32], xb[32];
      // every tensor-memory load of this warp has completed: the buffer may be refilled
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[bf]);
      };
      if (PASS == 1) {
        // this thread's window row: running max m and sum Z over the tile's keys,
        // chunk by chunk (chunks of keys at or beyond nvalid are skipped)
        const uint32_t hb = tbase + half * 128;
        const int r = half * 128 + quarter * 32 + lane;
        // four partial sums (independent add chains), combined in a fixed order
        float m = -INFINITY, Z4[4] = {0.f, 0.f, 0.f, 0.f};
        auto rescale = [&](float mx) {
          if (mx > m) {
            const float f = m == -INFINITY ? 0.f : ex2_approx((m - mx) * a.c);
#pragma unroll
            for (int q = 0; q < 4; ++q) Z4[q] *= f;
            m = mx;
          }
        };
        auto rowstats = [&](const float (&x)[32], int ch) {
          if (ch * 32 + 32 <= nvalid) {  // a full chunk (every tile but a row's last): no masks
            float mx = fmaxf(x[0], x[1]);
#pragma unroll
            for (int i = 2; i < 32; ++i) mx = fmaxf(mx, x[i]);
            rescale(mx);
            const float mc = m * a.c;
#pragma unroll
            for (int i = 0; i < 32; ++i) Z4[i & 3] += ex2_approx(fmaf(x[i], a.c, -mc));
          } else if (ch * 32 < nvalid) {
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (ch * 32 + i < nvalid) mx = fmaxf(mx, x[i]);
            rescale(mx);
            const float mc = m * a.c;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (ch * 32 + i < nvalid) Z4[i & 3] += ex2_approx(fmaf(x[i], a.c, -mc));
          }
        };
        tmem_ld32(hb, xa);
        tc_wait_ld_regs(xa);
        tmem_ld32(hb + 32, xb);
        rowstats(xa, 0);
        tc_wait_ld_regs(xb);
        tmem_ld32(hb + 64, xa);
        rowstats(xb, 1);
        tc_wait_ld_regs(xa);
        tmem_ld32(hb + 96, xb);
        rowstats(xa, 2);
        tc_wait_ld_regs(xb);
        release();
        rowstats(xb, 3);
        const float Z = (Z4[0] + Z4[1]) + (Z4[2] + Z4[3]);
        if (r < a.R) a.partial[(long long)u * a.R + r] = make_float2(m, Z);
      } else {
        // this thread's key: the sum over its half of the window rows of
        // exp2(x c - lse_r), chunk by chunk
        const int j = quarter * 32 + lane;
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};  // independent add chains, combined in a fixed order
        auto colsum = [&](const float (&x)[32], int ch) {
          const int col = ch * 32;
          const float* lc = lse_s + (ch - c_lo) * 32;
          if (col + 32 <= a.R) {  // a full chunk of window rows: no masks
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 l4 = *reinterpret_cast<const float4*>(lc + i);
              sum4[0] += ex2_approx(fmaf(x[i + 0], a.c, -l4.x));
              sum4[1] += ex2_approx(fmaf(x[i + 1], a.c, -l4.y));
              sum4[2] += ex2_approx(fmaf(x[i + 2], a.c, -l4.z));
              sum4[3] += ex2_approx(fmaf(x[i + 3], a.c, -l4.w));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              if (col + i < a.R) {
                const float4 l4 = *reinterpret_cast<const float4*>(lc + i);
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  if (col + i + q < a.R) sum4[q] += ex2_approx(fmaf(x[i + q], a.c, -lv[q]));
              }
            }
          }
        };
        tmem_ld32(tbase + c_lo * 32, xa);
        tc_wait_ld_regs(xa);
        for (int ch = c_lo; ch < c_hi; ch += 2) {  // xa holds chunk ch
          const bool has1 = ch + 1 < c_hi, has2 = ch + 2 < c_hi;
          if (has1) tmem_ld32(tbase + (ch + 1) * 32, xb);
          else release();
          colsum(xa, ch);
          if (has1) {
            tc_wait_ld_regs(xb);
            if (has2) tmem_ld32(tbase + (ch + 2) * 32, xa);
            else release();
            colsum(xb, ch + 1);
            if (has2) tc_wait_ld_regs(xa);
          }
        }
        float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        float* pb = part + (bf * 2 + ((it >> 1) & 1)) * kTileKeys;
        if (pair && half == 0) {  // hand the first half's sums to the second
          pb[j] = sum;
          named_bar_arrive(3 + bf, n_pair);
        } else {
          if (pair) {
            named_bar_sync(3 + bf, n_pair);
            sum = pb[j] + sum;  // first half + second half, in that order
          }
          if (j < nvalid) a.s[row_key_off(a.map, row) + (long long)tile * kTileKeys + j] = sum;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Softmax denominators of every (row, window row) from the tile partials.
__global__ void score_merge_kernel(const RowMap map, int R, int Rs, float c, const float2* __restrict__ partial,
                                   float* __restrict__ lse2) {
  const int row = blockIdx.x, r = threadIdx.x;
  if (r >= R) return;
  const int s = row / map.rows_per_seq;
  const int tpr = (map.L[s] + kTileKeys - 1) / kTileKeys;
  const long long u_first = map.tile_off[s] + (long long)(row - s * map.rows_per_seq) * tpr;
  float m = -INFINITY, Z = 0.f;
  for (int t = 0; t < tpr; ++t) {
    const float2 p = partial[(u_first + t) * R + r];
    if (p.x > m) {
      Z = Z * exp2f((m - p.x) * c) + p.y;
      m = p.x;
    } else {
      Z += p.y * exp2f((p.x - m) * c);
    }
  }
  lse2[(long long)row * Rs + r] = m * c + log2f(Z);
}

// fp32 inputs: row statistics of one 128-key tile on CUDA cores.
__global__ void score_f32_stats_kernel(const RowMap map, int R, int d, float c, const float* __restrict__ qwin,
                                       const float* __restrict__ K, float2* __restrict__ partial) {
  extern __shared__ float fs[];
  const int dp = d + 1;
  float* Ks = fs;                  // [128][d+1]
  float* Qs = fs + kTileKeys * dp;  // [R][d+1]
  const int u = blockIdx.x;
  int row, tile;
  tile_to_row(map, u, row, tile);
  const int nvalid = min(kTileKeys, row_len(map, row) - tile * kTileKeys);
  const float* Kt = K + (row_key_off(map, row) + (long long)tile * kTileKeys) * d;
  for (int i = threadIdx.x; i < kTileKeys * d; i += blockDim.x) {
    const int j = i / d, k = i % d;
    Ks[j * dp + k] = j < nvalid ? Kt[(long long)j * d + k] : 0.f;
  }
  const float* Qr = qwin + (long long)row * R * d;
  for (int i = threadIdx.x; i < R * d; i += blockDim.x) Qs[(i / d) * dp + i % d] = Qr[i];
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float m = -INFINITY, Z = 0.f;
    for (int j = 0; j < nvalid; ++j) {
      float x = 0.f;
      for (int k = 0; k < d; ++k) x = fmaf(Qs[r * dp + k], Ks[j * dp + k], x);
      if (x > m) {
        Z = Z * ex2_approx((m - x) * c) + 1.f;
        m = x;
      } else {
        Z += ex2_approx((x - m) * c);
      }
    }
    partial[(long long)u * R + r] = make_float2(m, Z);
  }
}

// fp32 inputs: column sums of one 128-key tile on CUDA cores.
__global__ void score_f32_colsum_kernel(const RowMap map, int R, int d, float c, const float* __restrict__ qwin,
                                        const float* __restrict__ K, const float* __restrict__ lse2,
                                        float* __restrict__ s) {
  extern __shared__ float fs[];
  const int dp = d + 1;
  float* Ks = fs;
  float* Qs = fs + kTileKeys * dp;
  float* Ls = Qs + R * dp;
  const int u = blockIdx.x;
  int row, tile;
  tile_to_row(map, u, row, tile);
  const int nvalid = min(kTileKeys, row_len(map, row) - tile * kTileKeys);
  const long long key0 = row_key_off(map, row) + (long long)tile * kTileKeys;
  const float* Kt = K + key0 * d;
  for (int i = threadIdx.x; i < kTileKeys * d; i += blockDim.x) {
    const int j = i / d, k = i % d;
    Ks[j * dp + k] = j < nvalid ? Kt[(long long)j * d + k] : 0.f;
  }
  const float* Qr = qwin + (long long)row * R * d;
  for (int i = threadIdx.x; i < R * d; i += blockDim.x) Qs[(i / d) * dp + i % d] = Qr[i];
  for (int i = threadIdx.x; i < R; i += blockDim.x) Ls[i] = lse2[(long long)row * ((R + 3) & ~3) + i];
  __syncthreads();
  const int j = threadIdx.x;
  if (j >= nvalid) return;
  float sum = 0.f;
  for (int r = 0; r < R; ++r) {
    float x = 0.f;
    for (int k = 0; k < d; ++k) x = fmaf(Qs[r * dp + k], Ks[j * dp + k], x);
    sum += ex2_approx(fmaf(x, c, -Ls[r]));
  }
  s[key0 + j] = sum;
}

}  // namespace

ScoreWs score_ws_layout(const RowMap& m, int R) {
  ScoreWs w;
  const long long tiles = m.tile_off[m.n_seq];
  w.status_off = 0;
  w.partial_off = 256;
  w.lse_off = w.partial_off + (((size_t)tiles * R * sizeof(float2) + 255) & ~size_t(255));
  w.bytes = w.lse_off + (((size_t)m.n_rows * ((R + 3) & ~3) * sizeof(float) + 255) & ~size_t(255));
  return w;
}

int launch_score(const kv_shape& sh, const RowMap& m, const void* qwin, const void* K, float* s, void* ws,
                 cudaStream_t st) {
  const int R = sh.group * sh.w;
  const int d = sh.head_dim;
  const ScoreWs lay = score_ws_layout(m, R);
  char* wsb = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(wsb + lay.status_off);
  float2* partial = reinterpret_cast<float2*>(wsb + lay.partial_off);
  float* lse2 = reinterpret_cast<float*>(wsb + lay.lse_off);
  const int total_tiles = m.tile_off[m.n_seq];
  const float c = (float)(1.4426950408889634 / std::sqrt((double)d));
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return KV_ERR_CUDA;
  const int merge_threads = ((R + 31) / 32) * 32;

  if (sh.dtype == KV_BF16) {
    CUtensorMap tmQ, tmK;
    if (!encode_rows_bf16(&tmQ, qwin, d, (long long)m.n_rows * R, kQRows)) return KV_ERR_CUDA;
    if (!encode_rows_bf16(&tmK, K, d, total_keys(m), kTileKeys)) return KV_ERR_CUDA;
    // per-device settings: made on every launch (cheap), for whichever device is current
    auto k1 = d == 128 ? score_tc_kernel<1, 2> : score_tc_kernel<1, 1>;
    auto k2 = d == 128 ? score_tc_kernel<2, 2> : score_tc_kernel<2, 1>;
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) != cudaSuccess ||
        cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) != cudaSuccess)
      return KV_ERR_CUDA;
    TcArgs a;
    a.map = m;
    a.R = R;
    a.Rs = (R + 3) & ~3;
    a.n2 = ((R + 15) / 16) * 16;
    a.total_tiles = total_tiles;
    a.c = c;
    a.partial = partial;
    a.lse2 = lse2;
    a.s = s;
    a.status = status;
    a.limit_ns = wait_limit_ns();
    const int grid = std::min(sm_count(), total_tiles);
    k1<<<grid, kThreads, kSmemAlloc, st>>>(tmQ, tmK, a);
    score_merge_kernel<<<m.n_rows, merge_threads, 0, st>>>(m, R, (R + 3) & ~3, c, partial, lse2);
    k2<<<grid, kThreads, kSmemAlloc, st>>>(tmQ, tmK, a);
  } else {
    const size_t sm1 = (size_t)(kTileKeys + R) * (d + 1) * sizeof(float);
    const size_t sm2 = sm1 + (size_t)R * sizeof(float);
    if (cudaFuncSetAttribute(score_f32_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(score_f32_colsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024) !=
            cudaSuccess)
      return KV_ERR_CUDA;
    const float* q = static_cast<const float*>(qwin);
    const float* Kf = static_cast<const float*>(K);
    score_f32_stats_kernel<<<total_tiles, 128, sm1, st>>>(m, R, d, c, q, Kf, partial);
    score_merge_kernel<<<m.n_rows, merge_threads, 0, st>>>(m, R, (R + 3) & ~3, c, partial, lse2);
    score_f32_colsum_kernel<<<total_tiles, 128, sm2, st>>>(m, R, d, c, q, Kf, lse2, s);
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace kvc
